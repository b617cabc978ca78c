"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects bad arguments on the host before anything is enqueued.

No call here reaches a kernel launch: every argument set is invalid in a way
the host-side validation catches first (pointers are fake but never used).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def L():
    from latent_kv_decode_b200 import build, ops
    if not os.path.exists(ops.LIB_PATH):
        build.build()
    return ops.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(mla_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("mla_absorb_q", "mla_decode", "mla_combine", "mla_up_proj"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from latent_kv_decode_b200 import ops
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(L, n), f"{n} declared in mla.h but not exported"
        assert n in ops._SIGS, f"{n} has no ctypes signature in the binding"


def test_status_strings(L):
    assert L.mla_status_string(0) == b"MLA_OK"
    assert L.mla_status_string(3) == b"MLA_ERR_WORKSPACE"
    assert L.mla_version().decode().count(".") == 2


@pytest.mark.parametrize("name,cls", [("mla_decode_args", "DecodeArgs"), ("mla_append_args", "AppendArgs"),
                                      ("mla_group_wo_args", "GroupWoArgs")])
def test_struct_layout_matches_header(name, cls):
    """ctypes mirror has the header's fields in the header's order."""
    from latent_kv_decode_b200 import ops
    src = open(HEADER).read()
    body = src[src.index(f"typedef struct {name} {{"):src.index(f"}} {name};")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for line in body.splitlines()[1:]:
        line = line.strip().rstrip(";")
        if not line:
            continue
        decl = re.sub(r"^(const\s+)?[\w]+\s*\**\s*", "", line)
        fields += [f.strip().lstrip("*") for f in decl.split(",")]
    assert fields == [f for f, _ in getattr(ops, cls)._fields_]


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails before any use


def _args(**over):
    from latent_kv_decode_b200 import ops
    a = ops.DecodeArgs()
    a.B, a.H, a.Q, a.Ckv, a.Dr = 2, 128, 1, 512, 64
    a.q_dtype = a.cache_dtype = ops.MLA_BF16
    a.q_lat = a.q_pe = a.kv_cache = a.pe_cache = a.x = FAKE
    a.kv_row_stride, a.pe_row_stride = 512, 64
    a.kv_batch_stride, a.pe_batch_stride = 512 * 100, 64 * 100
    a.Lk = 100
    a.softmax_scale = 0.07
    a.num_splits = 1
    for k, v in over.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,status", [
    (dict(q_lat=None), 1), (dict(kv_cache=None), 1), (dict(x=None), 1), (dict(q_pe=None), 1),
    (dict(Ckv=256), 2), (dict(Dr=48), 2), (dict(H=12), 2), (dict(H=256), 2), (dict(Q=5), 2),
    (dict(num_splits=-1), 1), (dict(num_splits=100000), 1), (dict(q_lat=FAKE + 8), 1),
    (dict(kv_row_stride=500), 1), (dict(kv_batch_stride=10), 1), (dict(softmax_scale=0.0), 1),
    (dict(cache_dtype=0), 2), (dict(rope_tail=32), 2), (dict(B=0), 1),
    (dict(cache_dtype=2), 2),                      # FP4 cache needs Dr == 0
    (dict(block_table=FAKE, page_size=0, max_pages=2, num_pages=4), 1),
    (dict(block_table=FAKE, page_size=64, max_pages=1, num_pages=4), 1),  # 64 < Lk
])
def test_decode_rejects_bad_arguments(L, over, status):
    a = _args(**over)
    assert L.mla_decode(ctypes.byref(a), None, 0, None) == status
    assert L.mla_combine(ctypes.byref(a), None, 0, None) == status
    assert L.mla_decode_num_splits(ctypes.byref(a)) == -1


def test_decode_rejects_missing_workspace(L):
    a = _args(num_splits=4)
    assert L.mla_decode_num_splits(ctypes.byref(a)) == 4
    need = L.mla_decode_workspace_size(ctypes.byref(a))
    assert need == ((4 * 2 * 128 * 512 * 4 + 255) // 256) * 256 + 4 * 2 * 128 * 4
    assert L.mla_decode(ctypes.byref(a), None, 0, None) == 3
    assert L.mla_decode(ctypes.byref(a), FAKE, need - 1, None) == 3
    assert L.mla_decode(ctypes.byref(a), FAKE + 16, need, None) == 3   # not 256-byte aligned
    assert L.mla_combine(ctypes.byref(a), None, 0, None) == 3


def test_single_split_needs_no_workspace(L):
    a = _args(num_splits=1)
    assert L.mla_decode_workspace_size(ctypes.byref(a)) == 0
    assert L.mla_combine(ctypes.byref(a), None, 0, None) == 0   # no-op with one split


@pytest.mark.parametrize("fn", ["mla_absorb_q", "mla_up_proj"])
@pytest.mark.parametrize("bad,status", [
    (dict(a=None), 1), (dict(a=FAKE + 4), 1), (dict(Dn=96), 2), (dict(Vd=64), 2),
    (dict(Ckv=256), 2), (dict(H=7), 2), (dict(dt=2), 2), (dict(B=-1), 1),
])
def test_projections_reject_bad_arguments(L, fn, bad, status):
    kw = dict(a=FAKE, w=FAKE, o=FAKE, B=2, H=128, Q=1, Dn=128, Vd=128, Ckv=512, dt=1)
    kw.update(bad)
    r = getattr(L, fn)(kw["a"], kw["w"], kw["o"], kw["B"], kw["H"], kw["Q"], kw["Dn"], kw["Vd"],
                       kw["Ckv"], kw["dt"], None)
    assert r == status


def test_ops_fail_loudly_without_library(monkeypatch, tmp_path):
    from latent_kv_decode_b200 import ops
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ops.MlaError):
        ops.lib()


def _append_args(**over):
    from latent_kv_decode_b200 import ops
    a = ops.AppendArgs()
    a.B, a.Q, a.Ckv, a.Dr = 2, 1, 512, 64
    a.src_dtype = a.cache_dtype = ops.MLA_BF16
    a.c_kv = a.k_pe = a.kv_cache = a.pe_cache = a.seq_lens = FAKE
    a.kv_row_stride, a.pe_row_stride = 512, 64
    a.kv_batch_stride, a.pe_batch_stride = 512 * 100, 64 * 100
    a.Lk = 100
    for k, v in over.items():
        setattr(a, k, v)
    return a


_FP4 = dict(cache_dtype=2, Dr=0, k_pe=None, pe_cache=None, kv_row_stride=288, kv_batch_stride=288 * 100)


@pytest.mark.parametrize("over,status", [
    (dict(c_kv=None), 1), (dict(kv_cache=None), 1), (dict(seq_lens=None), 1), (dict(k_pe=None), 1),
    (dict(B=0), 1), (dict(Q=0), 1), (dict(Lk=0), 1), (dict(src_dtype=2, cache_dtype=2), 2),
    (dict(src_dtype=0), 2),                              # float32 rows into a bf16 cache
    (dict(rope_tail=64), 2),                             # bf16 rope rows arrive rotated
    (dict(kv_row_stride=100), 1), (dict(kv_batch_stride=10), 1), (dict(seq_lens=FAKE + 2), 1),
    (dict(block_table=FAKE, page_size=64, max_pages=1, num_pages=4), 1),   # 64 < Lk
    (dict(block_table=FAKE, page_size=0, max_pages=2, num_pages=4), 1),
    (dict(_FP4, Ckv=256), 2), (dict(_FP4, Dr=64, k_pe=FAKE, pe_cache=FAKE), 2), (dict(_FP4, rope_tail=32), 2),
    (dict(_FP4, kv_row_stride=280), 1), (dict(_FP4, kv_row_stride=296), 1),
    (dict(_FP4, kv_cache=FAKE + 8), 1), (dict(_FP4, kv_batch_stride=288 * 100 + 8), 1),
    (dict(_FP4, rope_tail=64, rope_theta=0.0), 1),
])
def test_append_rejects_bad_arguments(L, over, status):
    a = _append_args(**over)
    assert L.mla_cache_append(ctypes.byref(a), None) == status


def _group_wo_args(**over):
    from latent_kv_decode_b200 import ops
    a = ops.GroupWoArgs()
    a.B, a.H, a.Q, a.Ckv, a.G, a.R, a.D, a.dtype = 32, 64, 1, 512, 8, 1024, 4096, 1
    a.x = a.wo_a = a.wo_b = a.out = FAKE
    for k, v in over.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,status", [
    (dict(x=None), 1), (dict(wo_a=None), 1), (dict(out=None), 1), (dict(B=0), 1), (dict(G=0), 1),
    (dict(R=0), 1), (dict(D=0), 1), (dict(x=FAKE + 8), 1), (dict(wo_b=FAKE + 2), 1),
    (dict(dtype=0), 2), (dict(G=3), 2), (dict(Ckv=96), 2), (dict(R=1000), 2), (dict(D=1000), 2),
    (dict(Q=17), 2),
])
def test_group_wo_rejects_bad_arguments(L, over, status):
    a = _group_wo_args(**over)
    assert L.mla_group_wo(ctypes.byref(a), None, 0, None) == status
    assert L.mla_group_wo_workspace_size(ctypes.byref(a)) == 0
