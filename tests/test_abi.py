"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments synchronously before any launch."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build():
    import kda_build as build
    build.build()


_build()
import gated_delta_rule_135_b200 as kda  # noqa: E402


def _declared_functions():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert "kda_fwd" in declared and "kda_fwd_staged" in declared
    lib = ctypes.CDLL(kda.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert declared <= set(kda.EXPORTED) | declared


def test_binding_fused_bound_matches_header():
    """The binding's fused-kernel clamp bound (used to label bench lines) is the header's."""
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    m = re.search(r"#define\s+KDA_FUSED_MIN_LOWER_BOUND\s+\(?\s*(-?[0-9.]+)f?\s*\)?", text)
    assert m, "KDA_FUSED_MIN_LOWER_BOUND not found in include/kda.h"
    assert float(m.group(1)) == kda.FUSED_MIN_LOWER_BOUND


def test_strerror_covers_every_status():
    for code, name in kda.STATUS_NAMES.items():
        assert kda.kda_strerror(code).startswith(name)
    assert kda.kda_strerror(99) == "KDA_ERR_UNKNOWN"
    assert re.match(r"^\d+\.\d+\.\d+$", kda.kda_version())


def _dims(H=2, T=256, hk=128, hv=128, batch=1, nseq=1):
    return kda.kda_dims(batch, T, H, nseq, hk, hv)


FAKE = 0x7F0000000000            # never dereferenced: validation fails first


def _call(dims, lb=-5.0, scale=0.088, base=FAKE, stride=1 << 28, cu=None, out=None,
          init=None, fin=None, misalign=None):
    p = [base + i * stride for i in range(8)]
    if misalign is not None:
        p[misalign] += 8
    q, k, v, g, beta, alog, dtb, o = p
    if out is not None:
        o = out
    return kda.lib().kda_fwd(q, k, v, g, beta, alog, dtb, ctypes.c_float(lb), ctypes.c_float(scale),
                             init, cu, o, fin, dims, None)


def test_rejects_unsupported_head_dims():
    assert _call(_dims(hk=64)) == 2
    assert _call(_dims(hv=256)) == 2


@pytest.mark.parametrize("lb", [0.5, float("nan")])
def test_rejects_bad_lower_bound(lb):
    assert _call(_dims(), lb=lb) == 1


@pytest.mark.parametrize("scale", [float("inf"), float("nan")])
def test_rejects_non_finite_scale(scale):
    assert _call(_dims(), scale=scale) == 1


def test_rejects_bad_dims():
    assert _call(_dims(H=0)) == 1
    assert _call(kda.kda_dims(1, -1, 2, 1, 128, 128)) == 1
    # cu_seqlens requires batch == 1
    assert _call(_dims(batch=2), cu=FAKE + (1 << 33)) == 1


@pytest.mark.parametrize("which", [0, 1, 2, 3, 5, 6, 7])
def test_rejects_misaligned_pointers(which):
    assert _call(_dims(), misalign=which) == 3


def test_beta_needs_only_element_alignment():
    # beta (index 4) is read element by element: +8 bytes passes validation (the call then
    # stops at the device check, with no GPU here); +2 bytes is rejected
    p = [FAKE + i * (1 << 28) for i in range(8)]
    p[4] += 2
    assert kda.lib().kda_fwd(*p[:7], ctypes.c_float(-5.0), ctypes.c_float(0.1), None, None, p[7], None,
                             _dims(), None) == 3
    p[4] += 6
    assert kda.lib().kda_fwd(*p[:7], ctypes.c_float(-5.0), ctypes.c_float(0.1), None, None, p[7], None,
                             _dims(), None) != 3


def test_rejects_output_aliasing_an_input():
    # out == q
    assert _call(_dims(), out=FAKE) == 1


def test_rejects_partially_overlapping_states():
    st = FAKE + (1 << 34)
    assert _call(_dims(), init=st, fin=st + 4096) == 1


def test_null_required_pointer():
    d = _dims()
    r = kda.lib().kda_fwd(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(-5.0),
                          ctypes.c_float(1.0), None, None, FAKE + (1 << 30), None, d, None)
    assert r == 1


def test_staged_workspace_layout_is_consistent():
    for varlen, dims in ((0, _dims(H=3, T=1000)), (1, _dims(H=96, T=8192, nseq=6))):
        L = kda.kda_staged_layout()
        assert kda.lib().kda_staged_workspace_layout(dims, varlen, ctypes.byref(L)) == 0
        T, H = dims.seqlen * (1 if varlen else dims.batch), dims.num_heads
        N = dims.num_seqs if varlen else dims.batch
        assert L.max_chunks == math.ceil(T / 64) + N
        offs = [L.chunk_table, L.gamma, L.w, L.u_tilde, L.p, L.u, L.chunk_states, L.total]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert L.gamma - L.chunk_table >= 16 * L.max_chunks + 4
        assert L.w - L.gamma >= 4 * T * H * 128
        assert L.u - L.p >= 4 * T * H * 64
        assert L.total - L.chunk_states >= 4 * L.max_chunks * H * 128 * 128
        assert kda.lib().kda_staged_workspace_size(dims, varlen) == L.total
        assert kda.lib().kda_fwd_workspace_size(dims) >= L.total


def test_decode_rejects_bad_arguments():
    lib = kda.lib()
    p = [FAKE + i * (1 << 28) for i in range(9)]
    call = lambda pp, lb=-5.0, scale=0.1, B=2, H=2: lib.kda_decode(  # noqa: E731
        *pp[:7], ctypes.c_float(lb), ctypes.c_float(scale), pp[7], pp[8], B, H, None)
    assert call(p, lb=1.0) == 1
    assert call(p, scale=float("inf")) == 1
    assert call(p, H=0) == 1
    assert call(p, B=-1) == 1
    bad = list(p)
    bad[3] += 4
    assert call(bad) == 3
    assert call(p[:8] + [p[0]]) == 1          # out aliases q
    assert call(p, B=0) == 0                  # nothing to do


def test_gdn_rejects_bad_arguments():
    assert kda.lib().kda_gdn_fwd(*([FAKE + i * (1 << 28) for i in range(7)]), ctypes.c_float(0.5),
                                 ctypes.c_float(0.1), None, None, FAKE + (7 << 28), None, _dims(), None) == 1
    assert kda.lib().kda_gdn_fwd(*([FAKE + i * (1 << 28) for i in range(7)]), ctypes.c_float(-1.0),
                                 ctypes.c_float(0.1), None, None, FAKE + (7 << 28), None, _dims(hk=64), None) == 2
    p = [FAKE + i * (1 << 28) for i in range(7)]
    p[3] += 2          # the scalar gate needs element (4-byte) alignment
    assert kda.lib().kda_gdn_fwd(*p, ctypes.c_float(-1.0), ctypes.c_float(0.1), None, None,
                                 FAKE + (7 << 28), None, _dims(), None) == 3


def _bwd_call(dims=None, grads_override=None, drop=None, dfinal=None, ws=None, ws_bytes=0):
    dims = dims or _dims()
    p = [FAKE + i * (1 << 28) for i in range(8)]          # q k v g beta A_log dt_bias d_out
    gp = [FAKE + (1 << 32) + i * (1 << 28) for i in range(8)]
    fields = dict(zip(kda.GRAD_NAMES, gp))
    fields.update(grads_override or {})
    if drop:
        fields[drop] = None
    gr = kda.kda_grads(*[fields[n] for n in kda.GRAD_NAMES])
    return kda.lib().kda_bwd(*p[:7], ctypes.c_float(-5.0), ctypes.c_float(0.1), None, None, p[7], dfinal,
                             ctypes.byref(gr), dims, ws, ctypes.c_size_t(ws_bytes), None)


def test_bwd_rejects_bad_arguments():
    lib = kda.lib()
    # no gradient block
    assert lib.kda_bwd(*([FAKE] * 7), ctypes.c_float(-5.0), ctypes.c_float(0.1), None, None, FAKE, None,
                       None, _dims(), None, ctypes.c_size_t(0), None) == 1
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias"):
        assert _bwd_call(drop=name) == 1, name
    base = FAKE + (1 << 32)
    assert _bwd_call(grads_override={"dq": base + 8}) == 3           # misaligned
    assert _bwd_call(grads_override={"dbeta": base + 4 * (1 << 28) + 2}) == 3
    assert _bwd_call(grads_override={"dq": FAKE}) == 1               # dq overlaps q
    assert _bwd_call(grads_override={"dk": base + 4096}) == 1         # dk overlaps dq
    assert _bwd_call(grads_override={"dA_log": FAKE + 7 * (1 << 28)}) == 1   # overlaps d_out
    dfin = FAKE + (1 << 34)
    assert _bwd_call(grads_override={"d_initial_state": dfin + 4096}, dfinal=dfin) == 1
    assert _bwd_call(dims=_dims(hk=64)) == 2
    assert _bwd_call(dims=_dims(H=0)) == 1


def test_bwd_argument_checks_pass_before_the_device_check():
    # valid arguments (beta-like dbeta at +4 bytes, d_initial aliasing d_final exactly, no
    # d_initial at all) get past validation: with no GPU here the call then fails the device
    # check (KDA_ERR_CUDA or KDA_ERR_UNSUPPORTED), never an argument error
    base = FAKE + (1 << 32)
    dfin = FAKE + (1 << 34)
    for kw in (dict(), dict(grads_override={"dbeta": base + 4 * (1 << 28) + 4}),
               dict(grads_override={"d_initial_state": dfin}, dfinal=dfin), dict(drop="d_initial_state")):
        assert _bwd_call(**kw) in (2, 4), kw


def test_bwd_workspace_extends_the_staged_layout():
    for varlen, dims in ((0, _dims(H=3, T=1000)), (1, _dims(H=96, T=8192, nseq=6))):
        T, H = dims.seqlen * (1 if varlen else dims.batch), dims.num_heads
        N = dims.num_seqs if varlen else dims.batch
        mc = math.ceil(T / 64) + N
        # T per chunk, dS' per chunk, dU dKhat d(gamma q) dW dGamma, dA per chunk, dgC, partials
        extra = 4 * (mc * H * 64 * 64 + mc * H * 128 * 128 + 5 * T * H * 128 + mc * H * 64 * 64
                     + mc * H * 128 + mc * H + mc * H * 128)
        staged = kda.lib().kda_staged_workspace_size(dims, varlen)
        assert kda.lib().kda_bwd_workspace_size(dims, varlen) >= staged + extra
        assert kda.lib().kda_bwd_workspace_size(dims, varlen) <= staged + extra + 16 * 256


def test_selftest_rejects_bad_limits():
    lib = kda.lib()
    assert lib.kda_selftest_wait_timeout(0, None, None) == 1                  # KDA_ERR_INVALID_ARG
    assert lib.kda_selftest_wait_timeout(2_000_000_000, None, None) == 1
    assert lib.kda_selftest_wait_timeout(1000, ctypes.c_void_p(FAKE + 2), None) == 3   # KDA_ERR_ALIGNMENT


def test_segment_query_leaves_varlen_batched_and_short_calls_unsplit():
    """kda_fwd_segments: only one fixed-layout sequence of at least 128 chunks is ever split (on
    a host without a GPU nothing is); varlen calls, batches and invalid dims get 1."""
    assert kda.kda_fwd_segments(2, 131072, varlen=True) == 1
    assert kda.kda_fwd_segments(2, 65536, batch=2) == 1
    assert kda.kda_fwd_segments(2, 128 * 64 - 1) == 1
    assert kda.kda_fwd_segments(0, 131072) == 1
    assert kda.kda_fwd_segments(32, 131072) >= 1
