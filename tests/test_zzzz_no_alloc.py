"""moe_permute_noalloc: the dispatch for callers that may not allocate device memory.

Some callers of this library cannot call cudaMalloc: a plugin or custom operator
inside a framework or inference server whose allocator owns the GPU, or a service
with a device-memory budget fixed at start-up.  For them moe_permute_noalloc keeps
its scratch in a fixed array inside the library instead of a caller workspace.
This test calls it through the C ABI twice in a row (a large call, then a smaller
one that leaves stale words of the first in the shared array) and compares every
output with moe_permute's, bit for bit (index maps and row copies are exact).
It is self-contained, so it passes alone in a fresh process and after the others.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _run_both(lib, _lib, T, E, k, D, seed):
    rng = np.random.default_rng(seed)
    ids = torch.from_numpy(np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)).cuda()
    x = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(torch.bfloat16).cuda()
    cfg = _lib.MoeConfig(D, 64, E, k, 7.0, 1.702, _lib.MOE_BF16, _lib.MOE_W_DENSE)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def outs():
        return (torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
                torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
                torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
                torch.zeros((T * k, D), dtype=torch.bfloat16, device="cuda"))

    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    a = outs()
    nws = lib.moe_permute_workspace_size(ctypes.byref(cfg), T)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    assert lib.moe_permute(ctypes.byref(cfg), T, p(ids), p(x), p(a[0]), p(a[1]), p(a[2]), p(a[3]), p(ws),
                           ws.numel(), stream) == _lib.MOE_OK
    b = outs()
    assert lib.moe_permute_noalloc(ctypes.byref(cfg), T, p(ids), p(x), p(b[0]), p(b[1]), p(b[2]), p(b[3]),
                                   stream) == _lib.MOE_OK
    torch.cuda.synchronize()
    assert lib.moe_last_device_error() == _lib.MOE_OK
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    return a


def test_noalloc_permute_matches_workspace_version():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_12_b200 import _lib, build
    build.build()
    lib = _lib.load()
    first = _run_both(lib, _lib, T=9000, E=128, k=4, D=64, seed=1)     # 128 x 36 chunks of scratch
    second = _run_both(lib, _lib, T=300, E=32, k=4, D=32, seed=2)      # smaller: stale words remain
    assert int(first[0][-1]) == 9000 * 4 and int(second[0][-1]) == 300 * 4


def test_noalloc_permute_takes_no_device_memory():
    """A call (after the first one on this device) leaves the device's free memory unchanged."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_12_b200 import _lib, build
    build.build()
    lib = _lib.load()
    T, E, k, D = 4096, 32, 4, 64
    rng = np.random.default_rng(3)
    ids = torch.from_numpy(np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)).cuda()
    x = torch.zeros((T, D), dtype=torch.bfloat16, device="cuda")
    outs = (torch.empty(E + 1, dtype=torch.int32, device="cuda"), torch.empty(T * k, dtype=torch.int32, device="cuda"),
            torch.empty(T * k, dtype=torch.int32, device="cuda"),
            torch.empty((T * k, D), dtype=torch.bfloat16, device="cuda"))
    cfg = _lib.MoeConfig(D, 64, E, k, 7.0, 1.702, _lib.MOE_BF16, _lib.MOE_W_DENSE)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    def call():
        assert lib.moe_permute_noalloc(ctypes.byref(cfg), T, p(ids), p(x), *(p(o) for o in outs), stream) == \
            _lib.MOE_OK
        torch.cuda.synchronize()

    call()                                   # the first call in this context looks up the array
    free_before, _ = torch.cuda.mem_get_info()
    call()
    free_after, _ = torch.cuda.mem_get_info()
    assert lib.moe_last_device_error() == _lib.MOE_OK
    assert free_after == free_before


def test_noalloc_permute_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_12_b200 import _lib, build
    build.build()
    lib = _lib.load()
    cfg = _lib.MoeConfig(64, 64, 256, 4, 7.0, 1.702, _lib.MOE_BF16, _lib.MOE_W_DENSE)
    dummy = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    T = 256 * 129                       # 256 experts x 129 chunks > 32768
    assert lib.moe_permute_noalloc(ctypes.byref(cfg), T, dummy, dummy, dummy, dummy, dummy, dummy, None) == \
        _lib.MOE_ERR_UNSUPPORTED
