"""Host I/O of a decode step on the GPU: basiskv_copy between device memory and
pinned host memory, the out-projection storing y straight into pinned host
memory, and the engine's host-buffer graph step against its device step.
The refusals are host-side checks (nothing is launched for them)."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from long_context_decode_basiskv_b200 import binding as bk  # noqa: E402
from long_context_decode_basiskv_b200.engine import DecodeEngine  # noqa: E402
from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink  # noqa: E402


@pytest.mark.parametrize("nbytes", [16, 4096, 96 * 1024, 1_000_003, 7])
def test_copy_round_trip(nbytes):
    g = torch.Generator().manual_seed(nbytes)
    src = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g)
    h_in = src.pin_memory()
    d = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    d2 = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    h_out = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
    bk.copy(d, h_in)          # host -> device
    bk.copy(d2, d)            # device -> device
    bk.copy(h_out, d2)        # device -> host
    torch.cuda.synchronize()
    assert torch.equal(d.cpu(), src)
    assert torch.equal(h_out, src)


def test_copy_refusals():
    L = bk.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    pageable = np.zeros(4096 + 64, dtype=np.uint8)
    off = (-pageable.ctypes.data) % 16                              # a 16-byte aligned pageable address
    pg = ctypes.c_void_p(pageable.ctypes.data + off)
    assert L.basiskv_copy(ctypes.c_void_p(d.data_ptr()), pg, 1024, s) == bk.ERR_INVALID_ARG
    assert L.basiskv_copy(pg, ctypes.c_void_p(d.data_ptr()), 1024, s) == bk.ERR_INVALID_ARG
    assert L.basiskv_copy(ctypes.c_void_p(d.data_ptr() + 1), ctypes.c_void_p(d.data_ptr() + 2048), 16, s) \
        == bk.ERR_INVALID_ARG                                       # misaligned
    assert L.basiskv_copy(ctypes.c_void_p(d.data_ptr()), ctypes.c_void_p(d.data_ptr() + 16), 1024, s) \
        == bk.ERR_INVALID_ARG                                       # overlapping
    assert L.basiskv_copy(None, ctypes.c_void_p(d.data_ptr()), 16, s) == bk.ERR_INVALID_ARG
    assert L.basiskv_copy(None, None, 0, s) == bk.OK                # nothing to do
    with pytest.raises(ValueError):
        bk.copy(d, torch.zeros(4096, dtype=torch.uint8))           # pageable CPU tensor
    torch.cuda.synchronize()


# the three out-projection kernels: mma.sync (bf16, batch <= 8), tcgen05 (a K too
# large for the mma kernel's shared memory), the fp32 one
SHAPES = [
    ("llama3_8b_32k", dict(batch=3, context=16 * 200 + 5, top_k=24)),
    ("llama3_70b_64k", dict(batch=2, context=16 * 150 + 9, top_k=20)),
    ("tiny_fp32", dict(batch=2, context=600, top_k=6)),
]


def _engine(base="llama3_8b_32k", kw=SHAPES[0][1], name="host_io"):
    wl = shrink(WORKLOADS[base], name=name, **kw)
    return DecodeEngine(make_case(wl, "cuda"))


@pytest.mark.parametrize("base,kw", SHAPES, ids=[s[0] for s in SHAPES])
def test_out_proj_into_pinned_host(base, kw):
    eng = _engine(base, kw)
    eng.step()
    torch.cuda.synchronize()
    hy = torch.full(tuple(eng.y.shape), float("nan"), dtype=torch.float32).pin_memory()
    eng.out_proj(y=hy)
    torch.cuda.synchronize()
    assert torch.equal(hy, eng.y.cpu())
    L = bk.lib()
    pageable = np.zeros(eng.y.numel() + 16, dtype=np.float32)
    off = ((-pageable.ctypes.data) % 16) // 4
    st = L.basiskv_out_proj(ctypes.byref(eng.cfg.c()), ctypes.byref(eng.factors.c()),
                            ctypes.c_void_p(eng.o_lat.data_ptr()), eng.y.shape[0],
                            ctypes.c_void_p(pageable.ctypes.data + 4 * off),
                            ctypes.c_void_p(eng.ws.data_ptr()), eng.ws.numel(),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bk.ERR_INVALID_ARG                                 # pageable y is refused
    assert not np.any(pageable)


@pytest.mark.parametrize("overlap", ["pdl", "streams"])
@pytest.mark.parametrize("base,kw", SHAPES, ids=[s[0] for s in SHAPES])
def test_graph_step_host_matches_device_step(base, kw, overlap):
    """The host-buffer graph step (inputs in by basiskv_copy, y stored on the host) gives
    exactly the device step's y, for the captured inputs and for new ones."""
    wl = shrink(WORKLOADS[base], name="host_io", **kw)
    eng = DecodeEngine(make_case(wl, "cuda"), overlap=overlap)
    hin = eng.input_buffer().cpu().pin_memory()
    hy = torch.zeros(tuple(eng.y.shape), dtype=torch.float32).pin_memory()
    eng.graph_step()
    torch.cuda.synchronize()
    ref = eng.y.clone()
    for _ in range(2):
        hy.zero_()
        eng.graph_step_host(hin, hy)
        torch.cuda.synchronize()
        assert int(eng.err.item()) == 0
        assert torch.equal(hy, ref.cpu())
    # new inputs: the host buffer is refilled in place, the captured graph replayed
    g = torch.Generator().manual_seed(7)
    fresh = (torch.randn(hin.shape, generator=g) * 0.5).to(hin.dtype)
    hin.copy_(fresh)
    eng.graph_step_host(hin, hy)
    torch.cuda.synchronize()
    got = hy.clone()
    eng.input_buffer().copy_(fresh.cuda())
    eng.step()
    torch.cuda.synchronize()
    assert int(eng.err.item()) == 0
    assert torch.equal(got, eng.y.cpu())
    assert not torch.equal(got, ref.cpu())
