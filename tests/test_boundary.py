"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function
include/sia.h declares, the ctypes structs match the C layout, and bad arguments are refused
on the host before anything is launched."""
import ctypes
import os
import subprocess

import pytest

import indexed_sparse_attention_paged_b200 as sia
from indexed_sparse_attention_paged_b200 import build as cuda_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    cuda_build.build()
    return sia.load_library()


def test_library_exports_every_declared_function(lib):
    names = sia.header_functions()
    assert {"sia_sparse_index_topk", "sia_sparse_mla_attend", "sia_fused_decode",
            "sia_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.sia_version() >= 100


def test_ctypes_structs_match_the_c_layout(tmp_path):
    fields = {"sia_index_args": sia.IndexArgs, "sia_attend_args": sia.AttendArgs,
              "sia_append_args": sia.AppendArgs}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "sia.h"', "int main(void) {"]
    for cname, cls in fields.items():
        lines.append('printf("%s %%zu\\n", sizeof(%s));' % (cname, cname))
        for f, _ in cls._fields_:
            lines.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (cname, f, cname, f))
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = dict(l.rsplit(" ", 1) for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.split("\n") if l)
    for cname, cls in fields.items():
        assert int(out[cname]) == ctypes.sizeof(cls)
        for f, _ in cls._fields_:
            assert int(out["%s.%s" % (cname, f)]) == getattr(cls, f).offset, (cname, f)


def test_status_strings(lib):
    assert lib.sia_status_string(0) == b"SIA_OK"
    assert lib.sia_status_string(2) == b"SIA_ERR_UNSUPPORTED"


def _index_args(**kw):
    a = sia.IndexArgs()
    a.batch, a.n_q, a.n_heads, a.head_dim, a.page_size = 2, 1, 64, 128, 64
    a.max_pages_per_seq, a.num_pages, a.top_k, a.dtype = 16, 32, 128, sia.SIA_BF16
    for name in ("q", "w", "k_cache", "page_table", "seq_lens", "topk_out"):
        setattr(a, name, 4096)   # never dereferenced: every case below fails on the host
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _attend_args(**kw):
    a = sia.AttendArgs()
    a.batch, a.n_q, a.n_heads, a.d_latent, a.d_rope = 2, 1, 128, 512, 64
    a.page_size, a.max_pages_per_seq, a.num_pages, a.top_k = 64, 16, 32, 128
    a.softmax_scale = 0.05
    for name in ("q", "kv_cache", "page_table", "seq_lens", "topk", "out"):
        setattr(a, name, 4096)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(batch=0), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(top_k=0), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(head_dim=48), sia.SIA_ERR_UNSUPPORTED),
    (dict(n_heads=65), sia.SIA_ERR_UNSUPPORTED),
    (dict(page_size=48), sia.SIA_ERR_UNSUPPORTED),
    (dict(dtype=7), sia.SIA_ERR_UNSUPPORTED),
    (dict(q=4100), sia.SIA_ERR_INVALID_ARGUMENT),          # misaligned
])
def test_index_arguments_refused_on_the_host(lib, kw, status):
    a = _index_args(**kw)
    assert lib.sia_sparse_index_topk(ctypes.byref(a), None, 0, None, None) == status
    assert lib.sia_last_error() != b""


@pytest.mark.parametrize("kw,status", [
    ({}, sia.SIA_ERR_INVALID_ARGUMENT),                      # scores_out is required
    (dict(scores_out=8192, q=None), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(scores_out=8192, head_dim=48), sia.SIA_ERR_UNSUPPORTED),
    (dict(scores_out=8200), sia.SIA_ERR_INVALID_ARGUMENT),    # misaligned scores_out
])
def test_scoring_only_arguments_refused_on_the_host(lib, kw, status):
    a = _index_args(**kw)
    assert lib.sia_index_scores(ctypes.byref(a), None, None) == status
    assert lib.sia_last_error() != b""


@pytest.mark.parametrize("kw,status", [
    (dict(out=None), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(d_latent=256), sia.SIA_ERR_UNSUPPORTED),
    (dict(n_heads=129), sia.SIA_ERR_UNSUPPORTED),
    (dict(softmax_scale=float("inf")), sia.SIA_ERR_INVALID_ARGUMENT),
])
def test_attend_arguments_refused_on_the_host(lib, kw, status):
    a = _attend_args(**kw)
    assert lib.sia_sparse_mla_attend(ctypes.byref(a), None, 0, None, None) == status


def test_fused_call_requires_matching_arguments(lib):
    for ia_kw, aa_kw in [(dict(top_k=64), {}), (dict(topk_out=8192), {}), (dict(batch=3), {}),
                         ({}, dict(page_table=8192)), ({}, dict(max_pages_per_seq=17))]:
        ia, aa = _index_args(**ia_kw), _attend_args(**aa_kw)
        st = lib.sia_fused_decode(ctypes.byref(ia), ctypes.byref(aa), None, 0, None, None)
        assert st == sia.SIA_ERR_INVALID_ARGUMENT, (ia_kw, aa_kw)
        assert b"same sequences" in lib.sia_last_error()


def test_workspace_sizes_follow_the_layout(lib):
    ia = _index_args()
    # scores: batch * n_q * max_pages * page_size fp32, rounded to 256 bytes
    assert lib.sia_index_workspace_size(ctypes.byref(ia)) == 2 * 1 * 16 * 64 * 4
    ia.scores_out = 8192
    assert lib.sia_index_workspace_size(ctypes.byref(ia)) == 0
    assert lib.sia_index_workspace_size(ctypes.byref(_index_args(batch=0))) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sia.index_args(q, q, q, q, q, top_k=4)


def test_wait_limit_setter_returns_the_previous_bound(lib):
    first = sia.set_wait_limit_ns(12345)
    assert sia.set_wait_limit_ns(0) == 12345
    assert sia.set_wait_limit_ns(first) == 2_000_000_000


def test_noalloc_entry_point_clears_a_stale_error_message(lib):
    bad = _index_args(batch=0)
    assert lib.sia_sparse_index_topk(ctypes.byref(bad), None, 0, None, None) == sia.SIA_ERR_INVALID_ARGUMENT
    assert lib.sia_last_error() != b""
    assert lib.sia_sparse_index_topk_noalloc(None, None, None) == sia.SIA_ERR_INVALID_ARGUMENT
    assert b"NULL" in lib.sia_last_error()


def _append_args(**kw):
    a = sia.AppendArgs()
    a.batch, a.n_q, a.head_dim, a.d_kv, a.page_size = 2, 1, 128, 576, 64
    a.max_pages_per_seq, a.num_pages = 16, 32
    a.key_format, a.kv_format = sia.SIA_KEY_BF16, sia.SIA_KV_BF16
    for name in ("new_k", "new_kv", "page_table", "seq_lens", "k_cache", "kv_cache"):
        setattr(a, name, 4096)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(new_k=None), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(batch=0), sia.SIA_ERR_INVALID_ARGUMENT),
    (dict(head_dim=48), sia.SIA_ERR_UNSUPPORTED),
    (dict(d_kv=2048), sia.SIA_ERR_UNSUPPORTED),
    (dict(key_format=5), sia.SIA_ERR_UNSUPPORTED),
    (dict(key_format=sia.SIA_KEY_FP8_POW2), sia.SIA_ERR_INVALID_ARGUMENT),   # k_scale missing
    (dict(kv_scale=8192), sia.SIA_ERR_INVALID_ARGUMENT),                    # scale for a bf16 cache
])
def test_append_arguments_refused_on_the_host(lib, kw, status):
    a = _append_args(**kw)
    assert lib.sia_cache_append(ctypes.byref(a), None, None) == status
    assert lib.sia_last_error() != b""
