"""The C ABI without a GPU: the library loads, exports every declared symbol, and rejects bad calls
on the host before launching anything."""
import ctypes
import glob
import os
import re

import pytest

import orthogonal_equivalence_cnp_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+char\s*\*|poetx_status|size_t|unsigned\s+long\s+long)\s+(poetx_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert len(declared) >= 11, declared
    so = ctypes.CDLL(P.library_path())
    for name in declared:
        assert hasattr(so, name), name
    assert set(declared) <= set(P.exported_symbols())


def test_status_strings():
    for code, name in P.STATUS.items():
        assert P.poetx_status_string(code) == name


def _desc(**kw):
    base = dict(d_in=256, d_out=256, b=32, k=3, dtype=P.POETX_F32, mode=P.POETX_FAST)
    base.update(kw)
    return P.poetx_desc(base["d_in"], base["d_out"], base["b"], base["k"], base["dtype"], base["mode"])


@pytest.mark.parametrize("kw,code", [
    (dict(b=48), 2), (dict(b=32, dtype=P.POETX_BF16), 2), (dict(d_in=250), 2), (dict(k=9), 2),
    (dict(k=-1), 1), (dict(dtype=7), 1), (dict(mode=3), 1), (dict(d_out=0), 1),
])
def test_invalid_descriptors_rejected(kw, code):
    d = _desc(**kw)
    assert P.poetx_workspace_size(d, 64) == 0
    L = P.lib()
    fake = 1 << 20  # aligned, never dereferenced: validation fails first
    st = L.poetx_cnp(ctypes.byref(d), fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == code


def test_onchip_cnp_needs_no_workspace_and_checks_alignment():
    # bf16 with b <= 256: the CNP forward and adjoint run on chip (no scratch); fp32 and b = 512
    # run through the GEMM kernels and need scratch.
    for b in (64, 128, 256):
        d = _desc(d_in=512, d_out=768, b=b, dtype=P.POETX_BF16)
        assert P.poetx_cnp_blocks_workspace_size(d, 1000) == 0
    assert P.poetx_cnp_blocks_workspace_size(_desc(d_in=1024, d_out=512, b=512, dtype=P.POETX_BF16), 4) > 0
    assert P.poetx_cnp_blocks_workspace_size(_desc(), 4) > 0
    L = P.lib()
    A = 1 << 20
    bf = _desc(d_in=512, d_out=768, b=256, dtype=P.POETX_BF16)
    ws = P.poetx_workspace_size(bf, 8)
    assert L.poetx_cnp(ctypes.byref(bf), A, A, A + 8, A, A, ws, None) == 3
    assert L.poetx_cnp(ctypes.byref(bf), A, None, A, A, A, ws, None) == 1
    assert L.poetx_cnp_blocks(ctypes.byref(bf), 3, A + 4, A, None, 0, None) == 3


def test_null_misaligned_and_workspace_errors():
    L = P.lib()
    d = _desc()
    ws = P.poetx_workspace_size(d, 64)
    assert ws > 0
    A = 1 << 20
    # NULL output
    assert L.poetx_forward(ctypes.byref(d), 64, A, A, A, A, A, A, None, A, A, ws, None) == 1
    # misaligned input
    assert L.poetx_forward(ctypes.byref(d), 64, A + 4, A, A, A, A, A, A, A, A, ws, None) == 3
    # workspace too small / missing
    assert L.poetx_forward(ctypes.byref(d), 64, A, A, A, A, A, A, A, A, A, 1024, None) == 4
    assert L.poetx_forward(ctypes.byref(d), 64, A, A, A, A, A, A, A, A, None, ws, None) == 4
    # mode / saved-buffer mismatch
    assert L.poetx_forward(ctypes.byref(d), 64, A, A, A, A, A, A, A, None, A, ws, None) == 1
    dm = _desc(mode=P.POETX_MEM)
    assert L.poetx_forward(ctypes.byref(dm), 64, A, A, A, A, A, A, A, A, A, ws, None) == 1
    # negative token count
    assert L.poetx_forward(ctypes.byref(d), -1, A, A, A, A, A, A, A, A, A, ws, None) == 1
    # zero tokens: valid, nothing launched
    assert L.poetx_forward(ctypes.byref(d), 0, A, A, A, A, A, A, A, A, A, ws, None) == 0
    # absorb must not alias
    assert L.poetx_absorb(ctypes.byref(d), A, A, A, A, None) == 1
    # merge with a NULL permutation
    assert L.poetx_merge(ctypes.byref(d), A, A, A, None, A, A, A, A, A, A, 1 << 30, None) == 1


def test_workspace_grows_with_tokens_and_mem_mode():
    d = _desc(d_in=4096, d_out=4096, b=256, dtype=P.POETX_BF16)
    a, b = P.poetx_workspace_size(d, 1024), P.poetx_workspace_size(d, 2048)
    assert 0 < a < b
    dm = _desc(d_in=4096, d_out=4096, b=256, dtype=P.POETX_BF16, mode=P.POETX_MEM)
    assert P.poetx_workspace_size(dm, 2048) > b


def test_gemm_hook_rejects_out_of_range_views():
    # A view that would read past its array is refused on the host.
    st = P.lib().poetx_test_gemm(0, 64, 64, 64, 2, 1, 1 << 20, 64, 64, 64, 64, 0, 0,
                                 1 << 20, 64, 64, 64, 0, 0, 0, 1 << 20, 0, 64, 0, 0, 0,
                                 1.0, 0.0, None, 0, 0, 0, 0, None)
    assert st == 1


def test_adamw_host_validation():
    L = P.lib()
    A = 1 << 20
    ok = P.poetx_adamw_cfg(1e-3, 0.5, 0.9, 0.999, 1e-8, 0.0)
    assert L.poetx_adamw_step(ctypes.byref(ok), 0, 1, A, A, A, A, None) == 0  # nothing to do
    assert L.poetx_adamw_step(ctypes.byref(ok), 16, 0, A, A, A, A, None) == 1  # t < 1
    assert L.poetx_adamw_step(ctypes.byref(ok), -1, 1, A, A, A, A, None) == 1
    assert L.poetx_adamw_step(ctypes.byref(ok), 16, 1, A, None, A, A, None) == 1
    assert L.poetx_adamw_step(ctypes.byref(ok), 16, 1, A, A, A + 4, A, None) == 3
    for bad in (P.poetx_adamw_cfg(1e-3, 0.5, 1.0, 0.999, 1e-8, 0.0), P.poetx_adamw_cfg(1e-3, 0.5, 0.9, 0.999, 0.0, 0.0),
                P.poetx_adamw_cfg(-1.0, 0.5, 0.9, 0.999, 1e-8, 0.0), P.poetx_adamw_cfg(1e-3, 0.5, 0.9, 0.999, 1e-8, -1.0)):
        assert L.poetx_adamw_step(ctypes.byref(bad), 16, 1, A, A, A, A, None) == 1
    assert L.poetx_adamw_reset(-1, A, A, None) == 1 and L.poetx_adamw_reset(0, None, None, None) == 0


def test_xq_host_validation():
    # POET-XQ: bf16 and mem mode only, d_in and d_out multiples of 256, pointers checked before
    # anything is launched.
    L = P.lib()
    A = 1 << 20
    good = P.poetx_desc(512, 768, 256, 3, P.POETX_BF16, P.POETX_MEM)
    fast = P.poetx_desc(512, 768, 256, 3, P.POETX_BF16, P.POETX_FAST)
    f32 = P.poetx_desc(512, 768, 256, 3, P.POETX_F32, P.POETX_MEM)
    odd = P.poetx_desc(384, 768, 128, 3, P.POETX_BF16, P.POETX_MEM)

    def fwd(d, codes=A, scales=A, ws_bytes=16):
        return L.poetx_xq_forward(ctypes.byref(d), 64, A, codes, scales, A, A, A, A, A, A, ws_bytes, None)

    assert fwd(fast) == 1 and fwd(f32) == 1 and fwd(odd) == 2
    assert fwd(good) == 4                      # workspace too small
    assert fwd(good, codes=None) == 1 and fwd(good, scales=A + 4) == 3
    assert L.poetx_xq_forward(ctypes.byref(good), 0, None, A, A, None, None, None, None, None, None, 0, None) == 0
    bwd = lambda d, ws_bytes=16: L.poetx_xq_backward(ctypes.byref(d), 64, A, A, A, A, A, A, A, A, A, A, A, A, A, A,
                                                     ws_bytes, None)
    assert bwd(fast) == 1 and bwd(odd) == 2 and bwd(good) == 4
    assert L.poetx_xq_quantize(ctypes.byref(fast), A, A, A, None) == 1
    assert L.poetx_xq_quantize(ctypes.byref(good), None, A, A, None) == 1
    assert L.poetx_xq_quantize(ctypes.byref(good), A, A, A + 8, None) == 3
    assert L.poetx_xq_dequantize(ctypes.byref(odd), A, A, A, None) == 2
    assert L.poetx_xq_merge(ctypes.byref(good), A, A, A, A, A, A, A, A, A, A, A, 16, None) == 4
    assert L.poetx_xq_merge(ctypes.byref(f32), A, A, A, A, A, A, A, A, A, A, A, 1 << 30, None) == 1


def test_check_permutation_on_the_host():
    import numpy as np
    P.poetx_check_permutation(np.random.default_rng(0).permutation(1000).astype(np.int32))
    P.poetx_check_permutation(np.zeros(0, np.int32))  # the bijection of the empty set
    for bad in ([0, 0, 2], [0, 1, 3], [-1, 0, 1], [2, 1]):
        with pytest.raises(P.PoetxError):
            P.poetx_check_permutation(np.array(bad, np.int32))
    assert P.lib().poetx_check_permutation(None, 3) == 1 and P.lib().poetx_check_permutation(None, 0) == 0
    assert P.lib().poetx_check_permutation(None, -1) == 1


def test_wait_probe_host_validation():
    L = P.lib()
    A = 1 << 20
    assert L.poetx_test_wait_timeout(1_000_000, None, None) == 1
    assert L.poetx_test_wait_timeout(10, A, None) == 1            # below 1 us
    assert L.poetx_test_wait_timeout(10 ** 9, A, None) == 1       # above 100 ms
    assert L.poetx_test_wait_timeout(1_000_000, A + 2, None) == 3


class _FakeCuda:
    """Stands in for a CUDA tensor in the binding's host-side checks (never reaches the library)."""

    def __init__(self, numel, dtype, contiguous=True):
        self._n, self.dtype, self._c = numel, dtype, contiguous
        self.is_cuda = True

    def numel(self):
        return self._n

    def is_contiguous(self):
        return self._c

    def data_ptr(self):
        return 1 << 20


def test_binding_checks_sizes_types_and_devices_before_calling():
    import numpy as np
    import torch
    d = _desc(d_in=512, d_out=256, b=256, dtype=P.POETX_BF16)
    P_ = 256 * 255 // 2
    good_t = _FakeCuda(P_ * 3, torch.float32)
    with pytest.raises(ValueError, match="theta"):
        P.poetx_cnp_blocks(d, 3, _FakeCuda(P_ * 3 - 1, torch.float32), _FakeCuda(3 * 256 * 256, torch.bfloat16), None)
    with pytest.raises(ValueError, match="Q"):
        P.poetx_cnp_blocks_noalloc(d, 3, good_t, _FakeCuda(3 * 256 * 256, torch.float32))
    with pytest.raises(ValueError, match="contiguous"):
        P.poetx_cnp_blocks(d, 3, good_t, _FakeCuda(3 * 256 * 256, torch.bfloat16, contiguous=False), None)
    with pytest.raises(ValueError, match="CUDA"):
        P.poetx_cnp_blocks(d, 3, torch.zeros(P_ * 3), _FakeCuda(3 * 256 * 256, torch.bfloat16), None)
    with pytest.raises(ValueError, match="X"):
        P.poetx_forward(d, 64, _FakeCuda(64 * 512 - 8, torch.bfloat16), None, None, None, None, None, None, None, None)
    with pytest.raises(ValueError, match="exceeds"):
        P.poetx_check_permutation(np.arange(4, dtype=np.int32), 5)
