"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the header
declares, and rejects bad arguments before any CUDA call (so these run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

import chunk_wise_hierarchical_summary_b200.hils as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "hils.h")).read()
    return sorted(set(re.findall(r"HILS_API\s+[\w\s\*]*?\b(hils_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) >= 10
    assert set(names) == set(H.EXPORTED)
    for n in names:
        assert hasattr(H.lib, n), n
    # and nothing else with the hils_ prefix is exported
    out = os.popen(f"nm -D --defined-only {H.LIB_PATH}").read()
    exported = {m.group(1) for m in re.finditer(r" T (hils_\w+)$", out, re.M)}
    assert exported == set(names)


def _header_prototypes():
    """(return type, [parameter types]) of every HILS_API function, comments stripped."""
    text = open(os.path.join(ROOT, "include", "hils.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    protos = {}
    for m in re.finditer(r"HILS_API\s+([\w\s\*]*?)\b(hils_\w+)\s*\(([^;{)]*)\)\s*;", text):
        ret, name, args = " ".join(m.group(1).split()), m.group(2), m.group(3).strip()
        params = [] if args in ("", "void") else [re.sub(r"\b\w+$", "", " ".join(a.split())).strip()
                                                  for a in args.split(",")]
        protos[name] = (ret, params)
    return protos


def _ctype_for(c_type: str):
    """The ctypes type the binding must give a header type: pointers and streams as void pointers, the
    params struct by pointer, integers by their width and sign, status enums as int."""
    if c_type == "const hils_params *":
        return ctypes.POINTER(H.Params)
    if c_type.endswith("*") or c_type == "hils_stream_t":
        return ctypes.c_void_p
    return {"size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32, "int": ctypes.c_int,
            "uint32_t": ctypes.c_uint32, "hils_status": ctypes.c_int}[c_type]


def test_binding_signatures_match_the_header():
    protos = _header_prototypes()
    assert set(protos) == set(H.EXPORTED)
    for name, (ret, params) in protos.items():
        f = getattr(H.lib, name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == len(params), name
        for i, (have, c_type) in enumerate(zip(f.argtypes, params)):
            assert have == _ctype_for(c_type), (name, i, c_type, have)
        want = ctypes.c_char_p if ret == "const char *" else _ctype_for(ret)
        assert f.restype == want, (name, ret, f.restype)
    # the params struct: ten int32 sizes, the float scale, the int32 dtype, in the header's order
    assert [n for n, _ in H.Params._fields_] == ["B", "T", "L", "Hq", "Hkv", "d", "S", "topk", "window",
                                                 "q_pos0", "scale", "dtype"]
    assert ctypes.sizeof(H.Params) == 12 * 4


def test_status_strings_and_version():
    for code, name in H.STATUS.items():
        assert H.lib.hils_status_string(code).decode() == name
    assert b"sm_100a" in H.lib.hils_version()


def P(**kw):
    base = dict(B=2, T=256, L=256, Hq=4, Hkv=2, d=128, S=64, topk=4, window=64, q_pos0=0, scale=0.0, dtype=0)
    base.update(kw)
    return H.Params(*[base[k] for k in ("B", "T", "L", "Hq", "Hkv", "d", "S", "topk", "window", "q_pos0")],
                    base["scale"], base["dtype"])


def test_workspace_sizes():
    assert H.workspace_size(P(), H.OP_SUMMARY) == 0
    assert H.workspace_size(P(), H.OP_SELECT) == 0
    assert H.workspace_size(P(), H.OP_ATTN_BWD) >= 2 * 4 * 256 * 4
    dec = P(B=8, T=1, L=524288, Hq=32, Hkv=8, topk=32, window=512, q_pos0=524287)
    assert 0 < H.workspace_size(dec, H.OP_DECODE) < 64 << 20
    assert H.lib.hils_workspace_size(ctypes.byref(P(Hq=3)), H.OP_SELECT) == ctypes.c_size_t(-1).value
    assert H.lib.hils_workspace_size(ctypes.byref(P()), 99) == ctypes.c_size_t(-1).value


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: validation fails first
ODD = ctypes.c_void_p(0x10008)


def attn(p, q=FAKE, out=FAKE, ws=None, nws=0):
    return H.lib.hils_attn_fwd(ctypes.byref(p) if p is not None else None, q, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               out, FAKE, ws, nws, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3), 1), (dict(B=0), 1), (dict(T=300), 1), (dict(q_pos0=-1), 1), (dict(dtype=7), 1),
    (dict(scale=-1.0), 1), (dict(d=96), 2), (dict(S=256), 2), (dict(topk=65), 2),
])
def test_invalid_sizes_rejected_before_launch(kw, status):
    assert attn(P(**kw)) == status
    assert H.lib.hils_last_error().decode().startswith("hils_attn_fwd")


def test_null_and_misaligned_pointers():
    assert attn(None) == 1
    assert attn(P(), q=None) == 1 and b"q is NULL" in H.lib.hils_last_error()
    assert attn(P(), out=ODD) == 1 and b"not 16-byte aligned" in H.lib.hils_last_error()


def test_decode_and_bwd_shape_rules():
    p = P(T=1, q_pos0=10)
    st = H.lib.hils_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None)
    assert st == 1 and b"q_pos0 == L-T" in H.lib.hils_last_error()
    p = P(T=1, q_pos0=255)
    st = H.lib.hils_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, None)
    assert st == 3  # workspace too small
    p = P(T=128, q_pos0=128)
    args = [FAKE] * 17
    st = H.lib.hils_attn_bwd(ctypes.byref(p), *args, 1 << 30, None)
    assert st == 1 and b"self-attention" in H.lib.hils_last_error()


def test_multi_token_decode_rules():
    # M = T query tokens at the end of the cache: 1 <= M <= 8 and q_pos0 == L - M
    p = P(T=9, q_pos0=256 - 9)
    st = H.lib.hils_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None)
    assert st == 1 and b"T <= 8" in H.lib.hils_last_error()
    p = P(T=4, q_pos0=256 - 3)
    st = H.lib.hils_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None)
    assert st == 1
    # M > 1 runs on the bf16 d 128 S 64 kernels only
    p = P(T=4, q_pos0=256 - 4, dtype=1)
    st = H.lib.hils_decode(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None)
    assert st == 2 and b"T=4 > 1 needs bf16" in H.lib.hils_last_error()
    # supported shape: the workspace grows with M
    one, four = P(T=1, L=65536, q_pos0=65535), P(T=4, L=65536, q_pos0=65532)
    n1 = H.lib.hils_workspace_size(ctypes.byref(one), H.OP_DECODE)
    n4 = H.lib.hils_workspace_size(ctypes.byref(four), H.OP_DECODE)
    assert n4 > 3 * n1 // 2
    st = H.lib.hils_decode(ctypes.byref(four), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, None)
    assert st == 3  # workspace too small: everything before it validated


def test_summary_range_checked():
    p = P()
    st = H.lib.hils_chunk_summary(ctypes.byref(p), FAKE, FAKE, 2, 5, FAKE, FAKE, None)
    assert st == 1 and b"chunk range" in H.lib.hils_last_error()


def test_shared_query_summary_checked():
    p = P()
    st = H.lib.hils_chunk_summary_shared_query(ctypes.byref(p), FAKE, FAKE, 2, 5, FAKE, FAKE, None)
    assert st == 1 and b"hils_chunk_summary_shared_query: chunk range" in H.lib.hils_last_error()
    st = H.lib.hils_chunk_summary_shared_query(ctypes.byref(p), FAKE, None, 0, 4, FAKE, FAKE, None)
    assert st == 1 and b"q_shared" in H.lib.hils_last_error()
    assert H.lib.hils_chunk_summary_shared_query(ctypes.byref(p), None, None, 3, 3, None, None, None) == 0


def test_fused_qcal_rules():
    p = P()
    st = H.lib.hils_select_topk_qcal(ctypes.byref(p), FAKE, FAKE, FAKE, 16, FAKE, FAKE, FAKE, None, None, None)
    assert st == 2 and b"rank 16" in H.lib.hils_last_error()
    p = P(dtype=1)
    st = H.lib.hils_select_topk_qcal(ctypes.byref(p), FAKE, FAKE, FAKE, 32, FAKE, FAKE, FAKE, None, None, None)
    assert st == 2 and b"hils_select_topk" in H.lib.hils_last_error()
    p = P()
    st = H.lib.hils_select_topk_qcal(ctypes.byref(p), FAKE, None, FAKE, 32, FAKE, FAKE, FAKE, None, None, None)
    assert st == 1 and b"w_down is NULL" in H.lib.hils_last_error()


def test_bsa_select_rules():
    p = P(topk=33)
    st = H.lib.hils_bsa_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, None)
    assert st == 2 and b"topk 33 > 32" in H.lib.hils_last_error()
    p = P(T=1, L=1 << 20, q_pos0=(1 << 20) - 1)
    st = H.lib.hils_bsa_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, None)
    assert st == 2 and b"> 1024" in H.lib.hils_last_error()
    p = P()
    st = H.lib.hils_bsa_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, None)
    assert st == 1 and b"mass is NULL" in H.lib.hils_last_error()
    st = H.lib.hils_bsa_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, ctypes.c_void_p(FAKE.value + 4), FAKE, None)
    assert st == 1 and b"gap is not 16-byte aligned" in H.lib.hils_last_error()


def test_select_too_many_chunks_for_one_cta():
    p = P(T=1, L=1 << 20, q_pos0=(1 << 20) - 1)
    st = H.lib.hils_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, None, None, 0, None)
    assert st == 2 and b"hils_decode" in H.lib.hils_last_error()


def test_select_shat_must_be_aligned():
    p = P()
    st = H.lib.hils_select_topk(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, ODD, None, 0, None)
    assert st == 1 and b"shat is not 16-byte aligned" in H.lib.hils_last_error()
    st = H.lib.hils_select_topk_qcal(ctypes.byref(P(T=128, L=128)), FAKE, FAKE, FAKE, 32, FAKE, FAKE, FAKE, None, ODD,
                                     None)
    assert st == 1 and b"shat is not 16-byte aligned" in H.lib.hils_last_error()


def attn_shat(p, idx=FAKE, shat=FAKE):
    return H.lib.hils_attn_fwd_shat(ctypes.byref(p), FAKE, FAKE, FAKE, idx, shat, FAKE, FAKE, None)


def test_attn_fwd_shat_rules():
    """The score-taking attention covers the tensor-core shapes only and checks its pointers on the host."""
    assert attn_shat(P(dtype=1)) == 2 and b"hils_attn_fwd" in H.lib.hils_last_error()
    assert attn_shat(P(d=64)) == 2
    assert attn_shat(P(topk=33)) == 2
    assert attn_shat(P(Hq=12, Hkv=4)) == 2  # 128 % G != 0
    assert attn_shat(P(), shat=None) == 1 and b"shat is NULL" in H.lib.hils_last_error()
    assert attn_shat(P(), idx=ODD) == 1 and b"idx is not 16-byte aligned" in H.lib.hils_last_error()


def test_wait_expiry_hook_rejects_limits_before_any_launch():
    """The failure-detection test hook validates its poll limit on the host (no CUDA call is made)."""
    assert H.lib.hils_test_wait_expiry(0, 0, None) == H.HilsError(1, "").status
    assert H.lib.hils_test_wait_expiry((1 << 20) + 1, 1, None) == 1
    assert b"max_polls" in H.lib.hils_last_error()
