"""Host-side checks of libgdn that need no GPU.

* the library loads and exports every entry point include/gdn.h declares;
* every argument check the C ABI documents returns its status code before
  anything is launched (the pointers used here are never dereferenced:
  each call is rejected by a scalar or pointer-value rule first).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    from gated_deltanet_state_gdn_b200 import build
    build.build()
    import gated_deltanet_state_gdn_b200 as g
    return g.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]*?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    syms = declared_symbols()
    assert {"gdn_prefill", "gdn_decode", "gdn_conv1d", "gdn_status_string"} <= set(syms)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    import gated_deltanet_state_gdn_b200 as g
    assert set(g.EXPORTED) == set(declared_symbols())


def test_abi_version_and_status_strings(L):
    assert L.gdn_abi_version() == 2
    import gated_deltanet_state_gdn_b200 as g
    for code, name in [(0, "GDN_OK"), (1, "GDN_ERR_NULL"), (2, "GDN_ERR_SHAPE"),
                       (3, "GDN_ERR_DTYPE"), (4, "GDN_ERR_ALIGN"), (5, "GDN_ERR_ALIAS"),
                       (6, "GDN_ERR_UNSUPPORTED"), (7, "GDN_ERR_CUDA")]:
        assert g.status_string(code) == name
    assert g.status_string(99) == "GDN_ERR_UNKNOWN"


# fake, never-dereferenced device addresses (distinct 256-byte aligned regions)
def P(i, off=0):
    return ctypes.c_void_p(0x7f0000000000 + i * (1 << 32) + off)


def prefill(L, **kw):
    args = dict(q=P(1), k=P(2), v=P(3), g=P(4), beta=P(5), alog=None, dtb=None, cu=None,
                init=None, final=P(7), out=P(8), B=2, N=64, Hq=1, Hv=1, Dk=16, Dv=16, dtype=0,
                scale=1.0, l2=0, flags=0, status=None, stream=None)
    args.update(kw)
    return L.gdn_prefill(args["q"], args["k"], args["v"], args["g"], args["beta"], args["alog"],
                         args["dtb"], args["cu"],
                         args["init"], args["final"], args["out"], args["B"], args["N"],
                         args["Hq"], args["Hv"], args["Dk"], args["Dv"], args["dtype"],
                         args["scale"], args["l2"], args["flags"], args["status"],
                         args["stream"])


def test_prefill_host_validation(L):
    assert prefill(L, dtype=5) == 3                       # GDN_ERR_DTYPE
    assert prefill(L, Hq=3, Hv=4) == 2                    # Hv % Hq != 0
    assert prefill(L, Dk=0) == 2
    assert prefill(L, Dk=300) == 6                        # beyond 256
    assert prefill(L, N=63) == 2                          # uniform packing needs N % B == 0
    assert prefill(L, q=None) == 1
    assert prefill(L, final=None) == 1
    assert prefill(L, beta=None) == 1
    assert prefill(L, v=P(3, 8)) == 4                     # 16-byte alignment
    assert prefill(L, g=P(4, 4)) == 4                     # g, beta: tensor-map bases
    assert prefill(L, beta=P(5, 8)) == 4
    assert prefill(L, g=P(4, 4), dtype=1, Hv=4, Dk=128, Dv=128) == 4
    assert prefill(L, g=P(4, 2)) == 4
    assert prefill(L, flags=1 << 9) == 6                  # unknown flag
    assert prefill(L, init=P(7, 256), final=P(7)) == 5    # initial/final overlap
    assert prefill(L, out=P(1, 64)) == 5                  # out overlaps q
    assert prefill(L, final=P(3, 16)) == 5                # final_state overlaps v
    assert prefill(L, B=0, N=0) == 0                      # nothing to do, nothing launched
    assert prefill(L, B=0, N=4) == 2


def test_prefill_rule_and_gate_validation(L):
    GATED, DELTA, LINEAR, QWEN, SIG = 1 << 3, 2 << 3, 3 << 3, 1 << 5, 1 << 6
    # decay input exactly for gated / gated_delta, beta exactly for delta / gated_delta
    assert prefill(L, flags=GATED) == 1                   # gated takes no beta
    assert prefill(L, flags=DELTA) == 1                   # delta takes no decay
    assert prefill(L, flags=LINEAR, beta=None) == 1
    assert prefill(L, g=None) == 1                        # gated_delta needs both
    # qwen needs a decay and both per-head vectors; sigmoid needs a beta
    assert prefill(L, flags=QWEN) == 1
    assert prefill(L, flags=QWEN, alog=P(9)) == 1
    assert prefill(L, flags=QWEN | DELTA, g=None, alog=P(9), dtb=P(10)) == 2
    assert prefill(L, flags=SIG | GATED, beta=None) == 2
    assert prefill(L, alog=P(9), dtb=P(10)) == 1          # vectors without the qwen gate
    assert prefill(L, flags=QWEN, alog=P(9, 2), dtb=P(10)) == 4
    assert prefill(L, flags=QWEN, alog=P(8, 4), dtb=P(10)) == 5   # out overlaps a_log
    assert prefill(L, dtype=2, flags=1 << 7) == 6         # unknown flag bit


def test_prefill_per_key_decay_validation(L):
    """GDN_DECAY_PER_KEY: g is [N, Hv, Dk]; it needs a rule with decay, and the overlap
    checks use the larger g."""
    import gated_deltanet_state_gdn_b200 as g
    PK, DELTA, LINEAR = g.GDN_DECAY_PER_KEY, 2 << 3, 3 << 3
    assert PK == 1 << 8
    assert prefill(L, flags=PK | DELTA, g=None) == 2      # no decay to spell per key
    assert prefill(L, flags=PK | LINEAR, g=None, beta=None) == 2
    # N * Hv * Dk floats of g = 64 * 16 * 4 bytes: out 4 KiB - 64 past g's start overlaps it
    assert prefill(L, flags=PK, out=P(4, 64 * 16 * 4 - 64)) == 5
    assert prefill(L, flags=PK, final=P(4, 64 * 16 * 4 - 64)) == 5
    assert prefill(L, flags=PK, g=P(4, 8)) == 4
    # bf16 heads of 8 to 128 run the per-key tensor-core kernel; fp16, fp32 and other heads the
    # per-token kernel; the sequence split never takes the per-key decay
    assert L.gdn_prefill_uses_chunked(g.GDN_BF16, 32, 128, 128, PK) == 1
    assert L.gdn_prefill_uses_chunked(g.GDN_BF16, 3, 12, 9, PK) == 1
    assert L.gdn_prefill_uses_chunked(g.GDN_F16, 3, 12, 9, PK) == 0
    assert L.gdn_prefill_uses_chunked(g.GDN_BF16, 3, 4, 128, PK) == 0   # narrower than 8
    assert L.gdn_prefill_uses_chunked(g.GDN_F32, 32, 128, 128, PK) == 0
    assert L.gdn_prefill_uses_chunked(g.GDN_BF16, 32, 160, 128, PK) == 0
    assert L.gdn_prefill_workspace_size(1, 32768, 16, 32, 128, 128, g.GDN_BF16, PK) == 0


def decode(L, **kw):
    args = dict(q=P(1), k=P(2), v=P(3), pool=P(4), P=16, ss=32 * 128 * 128, hs=128 * 128,
                ri=P(5), wi=None, si=None, A=P(6), a=P(7), dtb=P(8), b=P(9), scale=0.1,
                out=P(10), B=4, T=1, nh=1, H=32, HV=32, Dk=128, Dv=128, flags=0, status=None,
                stream=None)
    args.update(kw)
    return L.gdn_decode(args["q"], args["k"], args["v"], args["pool"], args["P"], args["ss"],
                        args["hs"], args["ri"], args["wi"], args["si"], args["A"], args["a"],
                        args["dtb"], args["b"], args["scale"], args["out"], args["B"],
                        args["T"], args["nh"], args["H"], args["HV"], args["Dk"], args["Dv"],
                        args["flags"], args["status"], args["stream"])


def test_decode_host_validation(L):
    assert decode(L, H=16) == 2                           # H != HV
    assert decode(L, T=17) == 6
    assert decode(L, nh=5) == 6
    assert decode(L, Dk=64) == 6
    assert decode(L, Dv=96) == 6
    assert decode(L, si=P(11), flags=2) == 2              # scatter + disable
    assert decode(L, hs=100) == 2                         # head stride below Dv*Dk
    assert decode(L, ss=16 * 128 * 128) == 2              # slot stride below HV*head_stride
    assert decode(L, ss=32 * 128 * 128 + 2) == 4          # stride not a multiple of 4 elements
    assert decode(L, pool=P(4, 8)) == 4                   # pool not 16-byte aligned
    assert decode(L, q=P(1, 4)) == 4
    assert decode(L, ri=None) == 1
    assert decode(L, b=None) == 1
    assert decode(L, out=P(4, 1024)) == 5                 # out inside the pool
    assert decode(L, flags=1 << 8) == 6                   # unknown flag
    assert decode(L, flags=1 << 7, ri=P(5, 4)) == 4       # int64 read slots need 8-byte alignment
    assert decode(L, flags=1 << 7, wi=P(11, 4)) == 4
    assert decode(L, P=0) == 2
    assert decode(L, B=0) == 0


def conv1d(L, **kw):
    args = dict(x=P(1), w=P(2), st=P(3), si=P(4), ro=P(5), out=P(6), B=2, N=64, C=64, K=4,
                S=8, dtype=1, ws=1, status=None, stream=None)
    args.update(kw)
    return L.gdn_conv1d(args["x"], args["w"], args["st"], args["si"], args["ro"], args["out"],
                        args["B"], args["N"], args["C"], args["K"], args["S"], args["dtype"],
                        args["ws"], args["status"], args["stream"])


def test_conv1d_host_validation(L):
    assert conv1d(L, dtype=7) == 3                        # GDN_ERR_DTYPE
    assert conv1d(L, K=0) == 2
    assert conv1d(L, K=9) == 6                            # kernel_size beyond 8
    assert conv1d(L, C=0) == 2
    assert conv1d(L, S=0) == 2                            # no slots
    assert conv1d(L, N=-1) == 2
    assert conv1d(L, N=1 << 31) == 6
    assert conv1d(L, x=None) == 1
    assert conv1d(L, si=None) == 1
    assert conv1d(L, ro=None) == 1
    assert conv1d(L, st=None) == 1                        # a window pool is needed for K > 1
    assert conv1d(L, x=P(1, 1)) == 4                      # bf16 elements need 2-byte alignment
    assert conv1d(L, dtype=0, out=P(6, 2)) == 4           # fp32 elements need 4-byte alignment
    assert conv1d(L, si=P(4, 2)) == 4
    assert conv1d(L, out=P(1, 128)) == 5                  # out overlaps x
    assert conv1d(L, st=P(6, 64)) == 5                    # pool overlaps out
    assert conv1d(L, st=P(2, 16)) == 5                    # pool overlaps the weights
    assert conv1d(L, B=0) == 0                            # nothing to do, nothing launched
    # a 1-tap convolution has no window, so the pool may be NULL; N = 0 launches nothing
    assert conv1d(L, K=1, st=None, N=0) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import gated_deltanet_state_gdn_b200._binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        b.lib()


def test_checked_build_exports_the_same_entry_points():
    """The bounds-checked test build (compiled with GDN_CHECKS) loads without a GPU and exports
    the same C ABI as the product library."""
    from gated_deltanet_state_gdn_b200 import build
    C = ctypes.CDLL(build.build(checked=True))
    for name in declared_symbols():
        assert hasattr(C, name), name
    C.gdn_abi_version.restype = ctypes.c_int32
    assert C.gdn_abi_version() == 2


def test_use_library_switches_and_fails_loudly(tmp_path):
    """use_library routes later calls through another build and returns the previous path; a
    missing library still raises instead of falling back."""
    import gated_deltanet_state_gdn_b200 as g
    import gated_deltanet_state_gdn_b200._binding as b
    prev = g.use_library(str(tmp_path / "missing.so"))
    try:
        with pytest.raises(RuntimeError, match="no fallback"):
            b.lib()
    finally:
        assert g.use_library(prev) == str(tmp_path / "missing.so")
    assert b.LIB_PATH == prev


def test_split_workspace_query_needs_a_device(L):
    """gdn_prefill_workspace_size is a host-only query; without a device (or for calls that
    never split) it is 0, and gdn_prefill_ws with a NULL workspace validates like gdn_prefill."""
    import gated_deltanet_state_gdn_b200 as g
    ws = L.gdn_prefill_workspace_size
    assert ws(1, 32768, 16, 32, 128, 128, g.GDN_F32, 0) == 0          # fp32: per-token kernel
    assert ws(1, 32768, 16, 32, 128, 128, g.GDN_BF16, g.GDN_PREFILL_SEQUENTIAL) == 0
    assert ws(1, 32768, 16, 32, 64, 64, g.GDN_BF16, 0) == 0           # only 128-wide heads
    assert ws(16, 32768, 16, 32, 128, 128, g.GDN_BF16, 0) == 0        # more than 8 requests
    assert ws(1, 32768, 3, 32, 128, 128, g.GDN_BF16, 0) == 0          # Hv % Hq != 0
    st = L.gdn_prefill_ws(P(1), P(2), P(3), P(4), P(5), None, None, None, None, P(7), P(8),
                          2, 64, 1, 1, 16, 16, 0, 1.0, 0, 0, None, 0, None, None)
    assert st == L.gdn_prefill(P(1), P(2), P(3), P(4), P(5), None, None, None, None, P(7), P(8),
                               2, 64, 1, 1, 16, 16, 0, 1.0, 0, 0, None, None)
