"""The C-ABI library without a GPU: it loads, exports every symbol that
include/hkv.h declares, and rejects bad arguments on the host."""
import ctypes
import os
import re

import pytest

import hash_sparse_kv_b200 as hkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hkv_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(hkv.lib_path):
        from hash_sparse_kv_b200 import build
        build.build()
    return hkv.lib()


def test_header_declares_the_bound_api():
    assert _declared() == sorted(hkv.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_version(lib):
    assert "sm_100a" in hkv.hkv_version()


def test_host_side_argument_errors(lib):
    h = hkv.hkv_hash(hkv.HKV_HASH_LSH, 64, 128, 0, hkv.HKV_BF16, 0, None, None, None, None, None)
    rc = lib.hkv_encode_keys(ctypes.byref(h), None, 10, 128, None, 4, None, None, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED and "head_dim" in hkv.hkv_last_error()
    h.head_dim = 128
    rc = lib.hkv_encode_keys(ctypes.byref(h), None, 10, 128, None, 4, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG  # R is NULL
    rc = lib.hkv_encode_keys(None, None, 10, 128, None, 4, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_retrieve_topk(1, 6, 4, 128, None, None, 10, 10, 0, 0, 4, None, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG and "multiple" in hkv.hkv_last_error()
    rc = lib.hkv_retrieve_topk(1, 4, 4, 96, None, None, 10, 10, 0, 0, 4, None, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED
    rc = lib.hkv_retrieve_topk(1, 4, 4, 128, None, None, 5, 10, 0, 0, 4, None, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG  # cap < n_tokens
    hs = hkv.hkv_hash(hkv.HKV_HASH_SIGN, 128, 128, 0, hkv.HKV_BF16, 0, None, None, None, None, None)
    rc = lib.hkv_append(ctypes.byref(hs), 1, 1, 4, None, None, None, None, None, None, 10, 8, None, None)
    assert rc == hkv.HKV_ERR_CAPACITY
    rc = lib.hkv_lse_merge(-1, 128, None, None, None, None, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_sparse_attend(1, 4, 4, 7, None, None, None, 10, 10, None, 0, 0, 0, 0.1, None, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG


def test_zero_sized_calls_are_noops(lib):
    h = hkv.hkv_hash(hkv.HKV_HASH_SIGN, 128, 128, 0, hkv.HKV_BF16, 0, None, None, None, None, None)
    assert lib.hkv_encode_keys(ctypes.byref(h), None, 0, 128, None, 4, None, None, None) == hkv.HKV_OK
    assert lib.hkv_retrieve_topk(0, 4, 4, 128, None, None, 10, 10, 0, 0, 4, None, None, None, 0, None, None) == hkv.HKV_OK
    assert lib.hkv_lse_merge(0, 128, None, None, None, None, None, None, None) == hkv.HKV_OK


def test_mlp_pack_sizes(lib):
    """Packed MLP weights: bf16 W1 [hidden_pad, 128] then fp16 W2 [bits, hidden_pad]."""
    assert lib.hkv_mlp_pack_bytes(512, 128) == 512 * 128 * 2 + 128 * 512 * 2
    assert lib.hkv_mlp_pack_bytes(200, 64) == 256 * 128 * 2 + 64 * 256 * 2
    assert lib.hkv_mlp_pack_bytes(0, 128) == 0
    assert lib.hkv_mlp_pack_bytes(2048, 128) == 0
    assert lib.hkv_mlp_pack_bytes(512, 96) == 0


def test_eviction_argument_errors(lib):
    rc = lib.hkv_evict_select(1, 4, 2, 96, None, None, 10, 10, 0, 0, None, None, None, 0, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED
    rc = lib.hkv_evict_select(1, 4, 3, 128, None, None, 10, 10, 0, 0, None, None, None, 0, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG  # 4 query heads do not split over 3 KV heads
    rc = lib.hkv_write_slots(1, 2, 7, 128, None, None, None, None, None, None, None, None, 10, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    assert lib.hkv_write_slots(0, 2, hkv.HKV_BF16, 128, None, None, None, None, None, None, None, None, 10, None,
                               None, None) == hkv.HKV_OK


def test_norm_weighted_and_split_argument_errors(lib):
    # norm-weighted retrieval: bad code width, NULL norms, too many candidates
    rc = lib.hkv_retrieve_topk_normw(1, 4, 2, 96, None, None, None, 10, 10, 0, 0, 4, None, None, None, 0, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED
    rc = lib.hkv_retrieve_topk_normw(1, 4, 2, 128, 1, 16, None, 10, 10, 0, 0, 4, 1, None, None, 0, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG  # norms is NULL
    rc = lib.hkv_retrieve_topk_normw(1, 4, 2, 128, 16, 16, 16, 70000, 70000, 0, 0, 4, 16, None, None, 0, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED and "workspace" in hkv.hkv_last_error()  # past 65536 without one
    rc = lib.hkv_retrieve_topk_normw(0, 4, 2, 128, None, None, None, 10, 10, 0, 0, 4, None, None, None, 0, None)
    assert rc == hkv.HKV_OK  # empty batch
    # norm-weighted decode step: 64-bit codes (sign codes are 128), NULL idx, empty batch
    rc = lib.hkv_decode_step_normw(1, 4, 2, hkv.HKV_BF16, 64, 16, 16, 16, 16, 16, 10, 10, 0, 0, 4, 0.1, None, 16,
                                   None, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED
    rc = lib.hkv_decode_step_normw(1, 4, 2, hkv.HKV_BF16, 128, 16, 16, 16, 16, 16, 10, 10, 0, 0, 4, 0.1, None, None,
                                   None, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    assert lib.hkv_decode_step_normw(0, 4, 2, hkv.HKV_BF16, 128, None, None, None, None, None, 10, 10, 0, 0, 4, 0.1,
                                     None, None, None, None, None, None, 0, None, None) == hkv.HKV_OK
    # no CUDA device here: the workspace size is 0 (the plan needs the SM count)
    assert lib.hkv_normw_workspace_bytes(1, 2, 200000, 0, 0, 8) == 0
    # token split: rank outside [0, G), NULL candidates
    rc = lib.hkv_split_select(2, 2, 1, 4, 2, 128, 8, None, None, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_split_select(2, 1, 1, 4, 2, 128, 8, None, None, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_split_select(2, 1, 1, 4, 2, 128, 0, None, None, None, None, None)
    assert rc == hkv.HKV_OK  # top_k 0
    # G-way merge: G 0, misaligned buffers
    rc = lib.hkv_lse_merge_n(0, 4, None, None, None, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_lse_merge_n(2, 4, 8, 16, 16, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG and "aligned" in hkv.hkv_last_error()
    rc = lib.hkv_lse_merge_n(2, 0, None, None, None, None, None)
    assert rc == hkv.HKV_OK


def test_paged_argument_errors(lib):
    # page_size 0, too few pages for n_tokens, NULL page table, too many candidates
    rc = lib.hkv_retrieve_topk_paged(1, 4, 2, 128, 16, 16, 16, 4, 4, 0, 10, 0, 0, 4, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG
    rc = lib.hkv_retrieve_topk_paged(1, 4, 2, 128, 16, 16, 16, 2, 4, 4, 10, 0, 0, 4, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG and "max_pages" in hkv.hkv_last_error()
    rc = lib.hkv_retrieve_topk_paged(1, 4, 2, 128, 16, 16, None, 4, 4, 4, 10, 0, 0, 4, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG and "page_table" in hkv.hkv_last_error()
    rc = lib.hkv_retrieve_topk_paged(1, 4, 2, 128, 16, 16, 16, 1000, 1000, 128, 70000, 0, 0, 4, 16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_UNSUPPORTED and "65536" in hkv.hkv_last_error()
    rc = lib.hkv_sparse_attend_paged(1, 4, 2, hkv.HKV_BF16, 16, 16, 16, 16, 2, 4, 4, 10, 16, 4, 0, 0, 0.088,
                                     16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG and "max_pages" in hkv.hkv_last_error()
    rc = lib.hkv_sparse_attend_paged(1, 4, 2, hkv.HKV_BF16, 16, 16, 16, 16, 4, 0, 4, 10, 16, 4, 0, 0, 0.088,
                                     16, None, None, 0, None, None)
    assert rc == hkv.HKV_ERR_INVALID_ARG  # num_pages 0


def test_binding_rejects_host_tensors_and_bad_shapes(lib):
    """The Python binding checks devices, dtypes and shapes before any call."""
    import torch
    q = torch.zeros(1, 4, 4, dtype=torch.int32)
    k = torch.zeros(1, 2, 64, 4, dtype=torch.int32)
    idx = torch.zeros(1, 2, 8, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        hkv.hkv_retrieve_topk(q, k, 64, 0, 0, 8, idx)
    with pytest.raises(ValueError, match="CUDA"):
        hkv.hkv_retrieve_topk_normw(q, k, torch.zeros(1, 2, 64, dtype=torch.float16), 64, 0, 0, 8, idx)
    with pytest.raises(ValueError, match="CUDA"):
        hkv.hkv_retrieve_topk_paged(q, torch.zeros(4, 2, 16, 4, dtype=torch.int32),
                                    torch.zeros(1, 4, dtype=torch.int32), 64, 0, 0, 8, idx)
    with pytest.raises(ValueError, match="CUDA"):
        hkv.hkv_split_select(0, 4, 128, torch.zeros(2, 1, 2, 8, dtype=torch.int32),
                             torch.zeros(2, 1, 2, 8, dtype=torch.int32), idx)
    with pytest.raises(ValueError, match="CUDA"):
        hkv.hkv_lse_merge_n(torch.zeros(2, 3, 128), torch.zeros(2, 3), torch.zeros(3, 128))


def test_plain_c_program_links_and_calls_the_library(lib, tmp_path):
    """include/hkv.h is valid C99 and libhkv.so links from C: a C program
    checks the host-side paths (no GPU needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_check"
    libdir = os.path.dirname(hkv.lib_path)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", libdir, "-lhkv", f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout
