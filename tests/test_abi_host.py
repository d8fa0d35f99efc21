"""Host-side checks of the C ABI: the library loads, exports every function include/*.h
declares, and rejects bad arguments before touching the GPU.  No compute call is made: every
call here fails validation (or is a documented no-op) before any CUDA API is reached, and the
pointers passed are never dereferenced on the host."""
import ctypes
import re
from pathlib import Path

import pytest

import entmax_tcgen05_tma_b200 as E

ROOT = Path(__file__).resolve().parents[1]


def _declared():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        for m in re.finditer(r"ENTMAX_API\s+[\w\s\*]+?\b(entmax_\w+)\s*\(", h.read_text()):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_abi():
    assert set(_declared()) == set(E.EXPORTED)


@pytest.mark.parametrize("name", _declared())
def test_library_exports(name):
    lib = ctypes.CDLL(str(E.LIB_PATH))
    assert hasattr(lib, name)


def test_strerror_and_version():
    assert E.strerror(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert E.strerror(code) != "unknown status"
    assert E.strerror(12345) == "unknown status"
    assert E.version() >= 100


def test_workspace_size():
    assert E.entmax_attn_bwd_workspace_size(0, 12, 128) == 0
    n = E.entmax_attn_bwd_workspace_size(4, 12, 4096)
    assert n >= 4 * 12 * 4096 * 4 and n % 256 == 0
    # rows of at most 512 keys take the tensor-core backward: the minimum (one float per row) is all
    # it asks for; longer rows get room for the support lists (the saved buffer) and the
    # support-list backward's buckets
    for B, H, L in ((2, 3, 1), (4, 12, 512), (1, 1, 300)):
        assert E.entmax_attn_bwd_workspace_size(B, H, L) == E.bwd_min_workspace_size(B, H, L)
    for B, H, L in ((4, 12, 4096), (1, 2, 513), (3, 5, 16384)):
        full = E.entmax_attn_bwd_workspace_size(B, H, L)
        assert full >= E.entmax_attn_saved_bytes(B, H, L) + E.entmax_attn_bwd_saved_workspace_size(B, H, L)
        assert full > E.bwd_min_workspace_size(B, H, L) and full % 256 == 0
        assert full < 1300 * B * H * L  # about 1.1 KB per query row


P = 0x10000  # fake, 16-byte aligned device address: never dereferenced by these calls


def _fwd(**kw):
    a = dict(Q=P, K=P, V=P, in_dtype=0, mask=None, causal=0, window=0, scale=0.125, B=1, H=1, L=64, D=64,
             O=P, out_dtype=0, tau=P, stream=None)
    a.update(kw)
    return E.lib.entmax_attn_fwd(a["Q"], a["K"], a["V"], a["in_dtype"], a["mask"], a["causal"], a["window"],
                                 a["scale"], a["B"], a["H"], a["L"], a["D"], a["O"], a["out_dtype"], a["tau"],
                                 a["stream"])


def _bwd(**kw):
    a = dict(Q=P, K=P, V=P, in_dtype=0, mask=None, causal=0, window=0, scale=0.125, B=1, H=1, L=64, D=64, tau=P,
             dO=P, dQ=P, dK=P, dV=P, ws=P, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return E.lib.entmax_attn_bwd(a["Q"], a["K"], a["V"], a["in_dtype"], a["mask"], a["causal"], a["window"],
                                 a["scale"], a["B"], a["H"], a["L"], a["D"], a["tau"], a["dO"], a["dQ"], a["dK"],
                                 a["dV"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(D=32), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(D=128), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(L=16385), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(B=300, H=300), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(window=32, causal=0), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(window=-1, causal=1), E.ENTMAX_ERR_ARG),
    (dict(causal=2), E.ENTMAX_ERR_ARG),
    (dict(in_dtype=7), E.ENTMAX_ERR_ARG),
    (dict(out_dtype=3), E.ENTMAX_ERR_ARG),
    (dict(scale=0.0), E.ENTMAX_ERR_ARG),
    (dict(scale=-0.125), E.ENTMAX_ERR_ARG),
    (dict(scale=float("nan")), E.ENTMAX_ERR_ARG),
    (dict(scale=float("inf")), E.ENTMAX_ERR_ARG),
    (dict(Q=None), E.ENTMAX_ERR_ARG),
    (dict(V=None), E.ENTMAX_ERR_ARG),
    (dict(O=None), E.ENTMAX_ERR_ARG),
    (dict(tau=None), E.ENTMAX_ERR_ARG),
    (dict(K=P + 8), E.ENTMAX_ERR_ARG),
    (dict(O=P + 4), E.ENTMAX_ERR_ARG),
    (dict(O=P + 8), E.ENTMAX_ERR_ARG),  # 16-byte stores
    (dict(B=-1), E.ENTMAX_ERR_ARG),
    (dict(B=0), E.ENTMAX_OK),
    (dict(L=0, Q=None, K=None, V=None, O=None, tau=None), E.ENTMAX_OK),
])
def test_fwd_argument_checks(kw, code):
    assert _fwd(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(D=16), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(window=4), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(tau=None), E.ENTMAX_ERR_ARG),
    (dict(dO=None), E.ENTMAX_ERR_ARG),
    (dict(dQ=None), E.ENTMAX_ERR_ARG),
    (dict(dV=None), E.ENTMAX_ERR_ARG),
    (dict(dO=P + 2), E.ENTMAX_ERR_ARG),
    (dict(dK=P + 4), E.ENTMAX_ERR_ARG),
    (dict(ws=None), E.ENTMAX_ERR_WORKSPACE),
    (dict(ws_bytes=64 * 4 - 1), E.ENTMAX_ERR_WORKSPACE),
    (dict(ws=P + 4), E.ENTMAX_ERR_ARG),
    (dict(B=0), E.ENTMAX_OK),
])
def test_bwd_argument_checks(kw, code):
    assert _bwd(**kw) == code


def _fwd_aux(**kw):
    a = dict(Q=P, K=P, V=P, in_dtype=0, mask=None, causal=0, window=0, scale=0.125, B=1, H=1, L=64, D=64,
             O=P, out_dtype=0, tau=P, Otil=P, rsum=P, stream=None)
    a.update(kw)
    return E.lib.entmax_attn_fwd_aux(a["Q"], a["K"], a["V"], a["in_dtype"], a["mask"], a["causal"], a["window"],
                                     a["scale"], a["B"], a["H"], a["L"], a["D"], a["O"], a["out_dtype"], a["tau"],
                                     a["Otil"], a["rsum"], a["stream"])


def _bwd_aux(**kw):
    a = dict(Q=P, K=P, V=P, in_dtype=0, mask=None, causal=0, window=0, scale=0.125, B=1, H=1, L=64, D=64, tau=P,
             Otil=P, rsum=P, dO=P, dQ=P, dK=P, dV=P, ws=P, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return E.lib.entmax_attn_bwd_aux(a["Q"], a["K"], a["V"], a["in_dtype"], a["mask"], a["causal"], a["window"],
                                     a["scale"], a["B"], a["H"], a["L"], a["D"], a["tau"], a["Otil"], a["rsum"],
                                     a["dO"], a["dQ"], a["dK"], a["dV"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [_fwd_aux, _bwd_aux])
@pytest.mark.parametrize("kw,code", [
    (dict(Otil=None), E.ENTMAX_ERR_ARG),
    (dict(rsum=None), E.ENTMAX_ERR_ARG),
    (dict(Otil=P + 8), E.ENTMAX_ERR_ARG),
    (dict(rsum=P + 2), E.ENTMAX_ERR_ARG),
    (dict(D=32), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(window=8), E.ENTMAX_ERR_UNSUPPORTED),
    (dict(B=0, Otil=None, rsum=None), E.ENTMAX_OK),
])
def test_aux_argument_checks(call, kw, code):
    assert call(**kw) == code


def test_binding_rejects_cpu_tensors():
    import torch

    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        E.entmax_attn_fwd(x, x, x)


def test_training_path_argument_checks():
    R = 64
    need = E.entmax_attn_saved_bytes(1, 1, R)
    assert need > R * 64 * 6 and E.entmax_attn_saved_bytes(0, 1, R) == 0
    assert E.entmax_attn_bwd_saved_workspace_size(1, 1, R) > R * 64 * 12
    f = E.lib.entmax_attn_fwd_train
    args = [P, P, P, 0, None, 0, 0, 0.125, 1, 1, R, 64, P, 0, P, P, need, None]
    assert f(*args[:16], need - 1, None) == E.ENTMAX_ERR_WORKSPACE
    assert f(*args[:15], None, need, None) == E.ENTMAX_ERR_WORKSPACE
    assert f(*args[:15], P + 16, need, None) == E.ENTMAX_ERR_ARG  # not 256-byte aligned
    bad = list(args)
    bad[11] = 32
    assert f(*bad) == E.ENTMAX_ERR_UNSUPPORTED
    b = E.lib.entmax_attn_bwd_saved
    ws = E.entmax_attn_bwd_saved_workspace_size(1, 1, R)
    bargs = [P, P, P, 0, None, 0, 0, 0.125, 1, 1, R, 64, P, P, need, P, P, P, P, P, ws, None]
    assert b(*bargs[:20], ws - 1, None) == E.ENTMAX_ERR_WORKSPACE
    nb = list(bargs)
    nb[13] = None
    assert b(*nb) == E.ENTMAX_ERR_WORKSPACE
    nb = list(bargs)
    nb[16] = P + 4
    assert b(*nb) == E.ENTMAX_ERR_ARG
    for k in (16, 17, 18):  # dQ, dK, dV take 16-byte stores
        nb = list(bargs)
        nb[k] = P + 8
        assert b(*nb) == E.ENTMAX_ERR_ARG
    assert f(*args[:12], P + 8, *args[13:]) == E.ENTMAX_ERR_ARG  # O of the training forward


def _gqa_calls(H, Hkv, in_dtype=0, B=1, L=64, D=64):
    """Status of the three grouped-query entry points for one head configuration."""
    R = max(B * H * L, 1)
    need = E.entmax_attn_saved_bytes(1, 1, R)
    ws = E.entmax_attn_bwd_saved_workspace_size(1, 1, R)
    f = E.lib.entmax_attn_fwd_gqa(P, P, P, in_dtype, None, 0, 0, 0.125, B, H, Hkv, L, D, P, 0, P, None)
    t = E.lib.entmax_attn_fwd_train_gqa(P, P, P, in_dtype, None, 0, 0, 0.125, B, H, Hkv, L, D, P, 0, P, P, need,
                                        None)
    b = E.lib.entmax_attn_bwd_saved_gqa(P, P, P, in_dtype, None, 0, 0, 0.125, B, H, Hkv, L, D, P, P, need, P, P, P,
                                        P, P, ws, None)
    return f, t, b


@pytest.mark.parametrize("H,Hkv,in_dtype,B,code", [
    (4, 3, 0, 1, E.ENTMAX_ERR_ARG),           # H not a multiple of H_kv
    (4, 0, 0, 1, E.ENTMAX_ERR_ARG),
    (4, -2, 0, 1, E.ENTMAX_ERR_ARG),
    (4, 8, 0, 1, E.ENTMAX_ERR_ARG),           # more key/value heads than query heads
    (0, 1, 0, 1, E.ENTMAX_ERR_ARG),
    (8, 2, 1, 1, E.ENTMAX_ERR_UNSUPPORTED),   # fp32 inputs with grouped heads
    (0, 0, 0, 1, E.ENTMAX_OK),
    (8, 2, 0, 0, E.ENTMAX_OK),                # empty batch: a no-op
])
def test_gqa_argument_checks(H, Hkv, in_dtype, B, code):
    assert _gqa_calls(H, Hkv, in_dtype, B) == (code, code, code)


def test_binding_rejects_bad_kv_head_count():
    import torch

    q = torch.zeros(1, 6, 8, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 4, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        E.entmax_attn_fwd_gqa(q, k, k)


def _ex_calls(alpha, B=1, H=2, Hkv=2, in_dtype=0, saved=P, saved_bytes=None, layout=0):
    R = max(B * H * 64, 1)
    need = E.entmax_attn_saved_bytes(1, 1, R) if saved_bytes is None else saved_bytes
    ws = E.entmax_attn_bwd_saved_workspace_size(1, 1, R)
    f = E.lib.entmax_attn_fwd_ex(P, P, P, in_dtype, None, 0, 0, 0.125, alpha, B, H, Hkv, 64, 64, layout, P, 0, P,
                                 saved, need, None)
    b = E.lib.entmax_attn_bwd_saved_ex(P, P, P, in_dtype, None, 0, 0, 0.125, alpha, B, H, Hkv, 64, 64, layout, P, P,
                                       need, P, P, P, P, P, ws, None)
    return f, b


@pytest.mark.parametrize("alpha,code", [
    (0.9998, E.ENTMAX_ERR_ARG),  # below the softmax band |alpha - 1| < 1e-4
    (0.5, E.ENTMAX_ERR_ARG),
    (2.0001, E.ENTMAX_ERR_ARG),
    (float("nan"), E.ENTMAX_ERR_ARG),
    (float("inf"), E.ENTMAX_ERR_ARG),
    (-1.5, E.ENTMAX_ERR_ARG),
])
def test_alpha_argument_checks(alpha, code):
    assert _ex_calls(alpha) == (code, code)


def test_ex_entry_points_validate_before_launch():
    # valid alpha, empty batch: a no-op
    assert _ex_calls(1.75, B=0) == (E.ENTMAX_OK, E.ENTMAX_OK)
    assert _ex_calls(2.0, B=0) == (E.ENTMAX_OK, E.ENTMAX_OK)
    # softmax: alpha = 1 and the band around it (the pages' |alpha - 1| < 1e-4)
    for a in (1.0, 0.99995, 1.00005):
        assert _ex_calls(a, B=0) == (E.ENTMAX_OK, E.ENTMAX_OK)
        assert _ex_calls(a, H=4, Hkv=3) == (E.ENTMAX_ERR_ARG, E.ENTMAX_ERR_ARG)
    # grouped heads are checked as in the _gqa calls
    assert _ex_calls(1.25, H=4, Hkv=3) == (E.ENTMAX_ERR_ARG, E.ENTMAX_ERR_ARG)
    assert _ex_calls(1.25, H=4, Hkv=2, in_dtype=1) == (E.ENTMAX_ERR_UNSUPPORTED, E.ENTMAX_ERR_UNSUPPORTED)
    # a saved buffer that is too small, or a size without a buffer
    f, _ = _ex_calls(1.25, saved_bytes=16)
    assert f == E.ENTMAX_ERR_WORKSPACE
    f, _ = _ex_calls(1.25, saved=None, saved_bytes=1 << 20)
    assert f == E.ENTMAX_ERR_WORKSPACE


def test_binding_rejects_bad_alpha_before_the_library():
    import torch

    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        E.entmax_attn_fwd_ex(q, q, q, alpha=1.5)  # CPU tensors are refused first


@pytest.mark.parametrize("layout", [-1, 2, 7])
def test_layout_argument_checks(layout):
    assert _ex_calls(1.5, layout=layout) == (E.ENTMAX_ERR_ARG, E.ENTMAX_ERR_ARG)
    assert _ex_calls(1.75, B=0, layout=1) == (E.ENTMAX_OK, E.ENTMAX_OK)


def test_binding_layout_detection():
    import torch

    from entmax_tcgen05_tma_b200 import _binding as bnd

    x = torch.zeros(2, 5, 3, 64)  # [B, L, H, D] memory
    assert bnd._layout_of(x.transpose(1, 2)) == E.ENTMAX_LAYOUT_BLHD
    assert bnd._layout_of(torch.zeros(2, 3, 5, 64)) == E.ENTMAX_LAYOUT_BHLD
    with pytest.raises(ValueError):
        bnd._layout_of(torch.zeros(2, 3, 64, 5).transpose(2, 3))  # d not innermost
    y = bnd._empty((2, 3, 5, 64), torch.float32, "cpu", E.ENTMAX_LAYOUT_BLHD)
    assert y.shape == (2, 3, 5, 64) and y.transpose(1, 2).is_contiguous()


def test_missing_library_fails_loudly():
    """No CPU path stands behind the binding: without the built library every call raises."""
    import subprocess
    import sys

    code = (
        "from pathlib import Path\n"
        "import entmax_tcgen05_tma_b200._binding as B\n"
        "B.LIB_PATH = Path('/nonexistent/libentmax_attn.so')\n"
        "for f in (B.version, lambda: B.strerror(0), lambda: B.entmax_attn_bwd_workspace_size(1, 1, 64)):\n"
        "    try:\n"
        "        f()\n"
        "    except ImportError as e:\n"
        "        assert 'not built' in str(e)\n"
        "    else:\n"
        "        raise SystemExit('call succeeded without the library')\n"
        "print('raised')\n"
    )
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0 and "raised" in r.stdout, r.stdout + r.stderr
