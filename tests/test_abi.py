"""The C-ABI library loads, exports every symbol include/rtp.h declares, the
ctypes binding declares every one with the header's argument list, and the
library rejects bad arguments before touching the GPU (runs without a GPU)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def rtp():
    from swa_hybrid_attention_b200 import build

    build.build()
    from swa_hybrid_attention_b200 import rtp as mod

    return mod


def declared_functions():
    text = open(os.path.join(ROOT, "include", "rtp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rtp_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(rtp):
    lib = ctypes.CDLL(rtp.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rtp.EXPORTED)


def test_status_strings(rtp):
    assert rtp.status_str(0) == "RTP_OK"
    assert rtp.status_str(1) == "RTP_ERR_INVALID_ARG"
    assert rtp.status_str(4) == "RTP_ERR_TIMEOUT"
    assert rtp.status_str(99) == "RTP_ERR_UNKNOWN"
    assert rtp.rtp_version() >> 16 == 1


BAD_CFGS = [
    dict(head_dim=64),
    dict(rank=8),
    dict(n_sink=2),
    dict(block=32),
    dict(seq=1000),  # not a multiple of block
    dict(n_q_heads=6, n_kv_heads=4),  # not a multiple
    dict(n_q_heads=12, n_kv_heads=4),  # odd group
    dict(n_q_heads=64, n_kv_heads=2),  # group > 16
    dict(window=0),
    dict(n_local=0),
    dict(topk=-1),
    dict(batch=0),
    dict(scale=-1.0),
]


@pytest.mark.parametrize("bad", BAD_CFGS)
def test_route_heads_rejects_bad_config(rtp, bad):
    args = dict(batch=1, seq=1024, n_q_heads=8, n_kv_heads=2, window=256, block=64, topk=4, n_local=2)
    extra = {k: v for k, v in bad.items() if k not in args}
    args.update({k: v for k, v in bad.items() if k in args})
    cfg = rtp.AttnConfig(**args)
    for k, v in extra.items():
        setattr(cfg, k, v)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_route_heads(cfg, [2, 0])
    assert e.value.status == rtp.RTP_ERR_INVALID_ARG


def test_route_heads_rejects_bad_kind(rtp):
    cfg = rtp.AttnConfig(1, 1024, 8, 2, 256, 64, 4, 2)
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_route_heads(cfg, [3, 0])
    assert e.value.status == rtp.RTP_ERR_INVALID_ARG


def test_decode_workspace_size_and_validation(rtp):
    cfg = rtp.AttnConfig(8, 1, 32, 4, 8192, 128, 32, 4)
    n = rtp.rtp_decode_workspace_bytes(cfg, [2, 2, 0, 2], 262144)
    # sel [8][4][37] int32 | cnt [8][4] int32 | one partial slot per span:
    # 8 sequences x (3 x 37 selected blocks + 8192 / 128 window pieces), each
    # [8 heads][132] fp32; every part rounded up to 256 bytes
    up = lambda x: (x + 255) // 256 * 256
    assert n == up(8 * 4 * 37 * 4) + up(8 * 4 * 4) + up(8 * (3 * 37 + 64) * 8 * 132 * 4)
    assert rtp.rtp_decode_workspace_bytes(cfg, [2, 2, 0, 5], 262144) == 0
    bad = rtp.AttnConfig(8, 1, 32, 4, 8192, 96, 32, 4)
    assert rtp.rtp_decode_workspace_bytes(bad, [2, 2, 0, 2], 262144) == 0
    with pytest.raises(rtp.RtpError) as e:
        rtp.rtp_sparse_decode(cfg, [2, 2, 0, 2], 262144, 0, 0, 0, 0, 0, 0, 0, 0)
    assert e.value.status == rtp.RTP_ERR_INVALID_ARG


def test_null_plan_is_rejected(rtp):
    for fn, nargs in [(rtp._lib.rtp_indexer_project, 7), (rtp._lib.rtp_block_select, 6),
                      (rtp._lib.rtp_hybrid_prefill, 8)]:
        assert fn(*([None] * nargs)) == rtp.RTP_ERR_INVALID_ARG
    assert rtp._lib.rtp_hybrid_prefill_items(None, None, None, None, None, None, None, 0, 0, 0,
                                             None) == rtp.RTP_ERR_INVALID_ARG
    assert rtp._lib.rtp_plan_num_local_items(None) == -1


def test_split_plan_rejects_key_begin_outside_the_range_start(rtp):
    """key_begin must lie in [0, q_begin]; refused before any device call."""
    cfg = rtp.AttnConfig(1, 1024, 8, 2, 256, 64, 4, 2)
    for q_begin, key_begin in [(256, 257), (256, -1), (0, 1)]:
        with pytest.raises(rtp.RtpError) as e:
            rtp.rtp_route_heads_split(cfg, [2, 0], q_begin, 512, key_begin)
        assert e.value.status == rtp.RTP_ERR_INVALID_ARG


def test_cache_calls_validate_before_launch(rtp):
    """Bad arguments are refused without touching the GPU (no device needed)."""
    cfg = rtp.AttnConfig(2, 1024, 8, 2, 256, 64, 4, 2)
    fake = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced on these paths
    lib = rtp._lib
    c = cfg.c()
    kinds = rtp._kinds([2, 0])
    inv = rtp.RTP_ERR_INVALID_ARG
    # append: pos outside [0, capacity)
    assert lib.rtp_cache_append(ctypes.byref(c), kinds, 1024, fake, fake, fake, fake, fake, fake, None) == inv
    assert lib.rtp_cache_append(ctypes.byref(c), kinds, -1, fake, fake, fake, fake, fake, fake, None) == inv
    # append: bad kind, null and unaligned pointers, missing centroids for a retrieval head
    assert lib.rtp_cache_append(ctypes.byref(c), rtp._kinds([3, 0]), 5, fake, fake, fake, fake, fake, fake,
                                None) == inv
    assert lib.rtp_cache_append(ctypes.byref(c), kinds, 5, None, fake, fake, fake, fake, fake, None) == inv
    assert lib.rtp_cache_append(ctypes.byref(c), kinds, 5, fake + 8, fake, fake, fake, fake, fake, None) == inv
    assert lib.rtp_cache_append(ctypes.byref(c), kinds, 5, fake, fake, fake, fake, fake, None, None) == inv
    # centroids: empty cache, bad block size
    assert lib.rtp_cache_centroids(ctypes.byref(c), kinds, 0, fake, fake, fake, None) == inv
    bad = rtp.AttnConfig(2, 1024, 8, 2, 256, 96, 4, 2).c()
    assert lib.rtp_cache_centroids(ctypes.byref(bad), kinds, 512, fake, fake, fake, None) == inv
    assert lib.rtp_cache_centroids(ctypes.byref(c), kinds, 512, None, fake, fake, None) == inv


def test_library_has_no_unresolved_internal_symbols(rtp):
    """Every kernel source is linked in (a missing one would leave rtp:: symbols undefined)."""
    import subprocess

    out = subprocess.run(["nm", "-D", "--undefined-only", rtp.LIB_PATH], capture_output=True, text=True).stdout
    assert "_ZN3rtp" not in out


def test_cluster_calls_validate_before_launch(rtp):
    cfg = rtp.AttnConfig(2, 4096, 8, 2, 256, 128, 4, 2)
    c = cfg.c()
    lib = rtp._lib
    fake = 1 << 20
    inv = rtp.RTP_ERR_INVALID_ARG
    good = dict(clu_end=2048, n_clusters=16)
    ptrs = [fake] * 9

    def cl(**kw):
        d = dict(good, **kw)
        return rtp.rtp_clusters(d["clu_end"], d["n_clusters"], *ptrs)

    kinds = rtp._kinds([2, 0])
    ws = rtp.rtp_cache_cluster_workspace_bytes(cfg, 2048)
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # projected keys, assignment, undecided-key list, one counter per head,
    # per-segment cluster counts (segments of 4096 keys, up to 2048 clusters)
    assert ws == (up(2 * 2 * 1920 * 16 * 4) + 2 * up(2 * 2 * 1920 * 4) + up(2 * 2 * 4) +
                  up(2 * 2 * 1 * 2048 * 4))
    for bad in (dict(clu_end=128), dict(clu_end=2000), dict(clu_end=8192), dict(n_clusters=0),
                dict(n_clusters=4096)):
        x = cl(**bad)
        assert lib.rtp_cache_cluster(ctypes.byref(c), kinds, 4, fake, fake, fake, ctypes.byref(x), fake, ws,
                                     None) == inv, bad
    x = cl()
    assert lib.rtp_cache_cluster(ctypes.byref(c), kinds, 0, fake, fake, fake, ctypes.byref(x), fake, ws, None) == inv
    assert lib.rtp_cache_cluster(ctypes.byref(c), kinds, 4, fake, fake, fake, ctypes.byref(x), fake, ws - 1,
                                 None) == inv
    # clustered decode: clustered rows beyond the cache, or a null clustering
    assert rtp.rtp_decode_clustered_workspace_bytes(cfg, [2, 0], 1024, 2048) == 0
    assert rtp.rtp_decode_clustered_workspace_bytes(cfg, [2, 0], 3000, 2048) > 0
    assert lib.rtp_sparse_decode_clustered(ctypes.byref(c), kinds, 3000, fake, fake, fake, fake, None, fake, fake,
                                           1 << 30, None, None, None) == inv


def declared_prototypes():
    """{name: (return type, [parameter types])} of every function in include/rtp.h."""
    text = open(os.path.join(ROOT, "include", "rtp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for ret, name, params in re.findall(r"([A-Za-z_][\w \*]*?)\s*\b(rtp_[a-z_]+)\s*\(([^;{]*?)\)\s*;", text):
        ps = [p.strip() for p in params.split(",") if p.strip()]
        if ps == ["void"]:
            ps = []
        types = [re.sub(r"\s*\b\w+$", "", p) if not p.endswith("*") else p for p in ps]
        out[name] = (ret.strip(), types)
    return out


def _kind_of_c(t: str) -> str:
    t = t.replace("const", "").strip()
    if "*" in t:
        return "ptr"
    return {"int": "int", "long": "long", "size_t": "size_t", "float": "float", "double": "double",
            "unsigned": "uint", "rtp_status": "int", "void": "void"}[t]


def _kind_of_ctypes(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_long: "long", ctypes.c_size_t: "size_t", ctypes.c_float: "float",
            ctypes.c_double: "double", ctypes.c_uint: "uint"}[t]


def test_binding_signatures_match_the_header(rtp):
    """ctypes does not check a call against the C prototype, so the binding's
    argument list is compared with rtp.h here: same count, and each argument
    of the same kind (pointer, int, long, size_t, float, unsigned), and the
    same kind of result."""
    protos = declared_prototypes()
    assert set(protos) == set(rtp.EXPORTED)
    for name, (ret, params) in protos.items():
        f = getattr(rtp._lib, name)
        got = [_kind_of_ctypes(t) for t in (f.argtypes or [])]
        assert got == [_kind_of_c(p) for p in params], (name, got, params)
        assert _kind_of_ctypes(f.restype) == _kind_of_c(ret), (name, f.restype, ret)


def declared_structs():
    """{typedef name: [(field type, field name)]} of the header's plain structs."""
    text = open(os.path.join(ROOT, "include", "rtp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for body, name in re.findall(r"typedef struct\s*\{(.*?)\}\s*(\w+)\s*;", text, flags=re.S):
        fields = []
        for decl in body.split(";"):
            decl = " ".join(decl.split())
            if decl:
                m = re.match(r"(.*?)(\w+)$", decl)
                fields.append((m.group(1).strip(), m.group(2)))
        out[name] = fields
    return out


def test_binding_structs_match_the_header(rtp):
    """The ctypes structures passed by pointer have the header's fields, in
    its order and of its kinds, and the same size."""
    structs = declared_structs()
    assert set(structs) == {"rtp_attn_cfg", "rtp_clusters"}
    for name, fields in structs.items():
        cls = getattr(rtp, name)
        got = [(n, _kind_of_ctypes(t)) for n, t in cls._fields_]
        assert got == [(n, _kind_of_c(t)) for t, n in fields], name
    assert ctypes.sizeof(rtp.rtp_attn_cfg) == 12 * 4
