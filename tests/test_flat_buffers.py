"""Host logic of the flat step buffers (one copy moves every input, one every
output): alignment, sizes and independence of the views."""
import torch

from fp4_sparse_attention_csa2_b200.runner import FLAT_ALIGN, flat_views


def test_views_are_aligned_disjoint_and_typed():
    specs = [((1, 1, 64, 512), torch.bfloat16), ((1, 1, 32, 64), torch.bfloat16), ((1, 1, 32), torch.float32),
             ((3,), torch.int32), ((1, 1, 64, 512), torch.float32), ((1, 1, 7), torch.float32)]
    buf, views = flat_views(specs, "cpu")
    base = buf.data_ptr()
    spans = []
    for v, (shape, dtype) in zip(views, specs):
        assert tuple(v.shape) == shape and v.dtype == dtype and v.is_contiguous()
        off = v.data_ptr() - base
        assert off % FLAT_ALIGN == 0
        spans.append((off, off + v.numel() * v.element_size()))
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0                                  # in order, no overlap
    assert spans[-1][1] <= buf.numel()
    for i, v in enumerate(views):
        v.fill_(i + 1)
    for i, v in enumerate(views):
        assert torch.all(v == i + 1)                     # no view wrote into another


def test_buffer_round_trip_moves_every_view():
    specs = [((5, 3), torch.float32), ((17,), torch.bfloat16), ((2, 2), torch.int32)]
    src, sv = flat_views(specs, "cpu")
    dst, dv = flat_views(specs, "cpu")
    g = torch.Generator().manual_seed(0)
    for v in sv:
        v.copy_(torch.randint(-100, 100, v.shape, generator=g).to(v.dtype))
    dst.copy_(src)                                       # one copy of the whole buffer
    for a, b in zip(sv, dv):
        assert torch.equal(a, b)
