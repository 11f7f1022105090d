"""The pins catch plausible slips: each case below plants one mistake in the
oracle (on the CPU, through monkeypatch) and checks that at least one pin
fails.  A pin set that still passed with the mistake in place would not be
pinning that part of the oracle."""
import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins


def _fails(*checks):
    """True when at least one of the pin calls raises AssertionError."""
    failed = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            failed += 1
    return failed > 0


# -- mutations of the norm-weighted score -----------------------------------

def _normw_with(score_fn, largest_first=True):
    def retrieve_normw(q_codes, k_codes, norms, N, n_sink, n_local, top_k):
        q_codes = np.asarray(q_codes, dtype=np.uint32)
        k_codes = np.asarray(k_codes, dtype=np.uint32)
        norms = np.asarray(norms, dtype=np.float16)
        B, Hq, W = q_codes.shape
        Hkv = k_codes.shape[1]
        g = Hq // Hkv
        lo, hi = oracle.candidate_range(N, n_sink, n_local)
        idx = np.full((B, Hkv, top_k), -1, dtype=np.int64)
        score = np.full((B, Hkv, top_k), -np.inf)
        for b in range(B):
            for kh in range(Hkv):
                D = oracle.hamming(q_codes[b, kh * g:(kh + 1) * g], k_codes[b, kh, :N])
                S = score_fn(oracle.as_f64(norms[b, kh, :N]), D, g, 32 * W)
                sel = oracle.select_topk(-S if largest_first else S, lo, hi, top_k)
                idx[b, kh, : sel.size] = sel
                score[b, kh, : sel.size] = S[sel]
        return idx, score
    return retrieve_normw


def _normw_pins():
    return [lambda c=c: pins.test_normw_fixture(c) for c in "abcd"] + [
        lambda: pins.test_normw_score_is_norm_times_sign_inner_product(0),
        lambda: pins.test_normw_brute_force(3),
        pins.test_normw_equal_norms_is_hamming_retrieval,
        pins.test_normw_norm_scaling_and_zero_norms,
    ]


@pytest.mark.parametrize("name,fn,largest", [
    ("factor 2 dropped", lambda n, D, g, b: n * (g * b - D), True),
    ("group size dropped", lambda n, D, g, b: n * (b - 2 * D), True),
    ("norm ignored", lambda n, D, g, b: 1.0 * (g * b - 2 * D), True),
    ("norm squared", lambda n, D, g, b: n * n * (g * b - 2 * D), True),
    ("smallest first", lambda n, D, g, b: n * (g * b - 2 * D), False),
])
def test_normw_mutations_fail_a_pin(monkeypatch, name, fn, largest):
    monkeypatch.setattr(oracle, "retrieve_normw", _normw_with(fn, largest))
    assert _fails(*_normw_pins()), name


# -- mutations of the page gather --------------------------------------------

def _gather_with(page_of, slot_of):
    def gather_pages(pool, page_table, page_size, N):
        table = np.asarray(page_table, dtype=np.int64)
        pool = np.asarray(pool)
        out = np.empty((table.shape[0], pool.shape[1], N) + pool.shape[3:], dtype=pool.dtype)
        for b in range(table.shape[0]):
            for t in range(N):
                out[b, :, t] = pool[int(table[b, page_of(t, page_size) % table.shape[1]]), :,
                                    slot_of(t, page_size) % page_size]
        return out
    return gather_pages


@pytest.mark.parametrize("name,page_of,slot_of", [
    ("page from the slot", lambda t, P: t % P, lambda t, P: t // P),
    ("next page", lambda t, P: t // P + 1, lambda t, P: t % P),
    ("slot reversed", lambda t, P: t // P, lambda t, P: P - 1 - t % P),
])
def test_gather_mutations_fail_a_pin(monkeypatch, name, page_of, slot_of):
    monkeypatch.setattr(oracle, "gather_pages", _gather_with(page_of, slot_of))
    assert _fails(pins.test_gather_pages_identity_table_is_a_reshape, pins.test_gather_pages_permuted_table,
                  pins.test_paged_retrieval_equals_contiguous_retrieval), name


# -- mutations of the shared steps ---------------------------------------------

def test_ties_to_the_highest_index_fail_a_pin(monkeypatch):
    def select_topk(D, lo, hi, k):
        if hi <= lo or k <= 0:
            return np.zeros(0, dtype=np.int64)
        cand = np.arange(lo, hi, dtype=np.int64)
        order = np.lexsort((-cand, D[lo:hi]))  # equal D: highest index first
        return np.sort(cand[order[: min(k, hi - lo)]])
    monkeypatch.setattr(oracle, "select_topk", select_topk)
    assert _fails(pins.test_topk_fixture, lambda: pins.test_topk_brute_force_rank(0))


def test_first_head_only_fails_a_pin(monkeypatch):
    def hamming(q_codes, k_codes):
        q = np.asarray(q_codes, dtype=np.uint32)
        k = np.asarray(k_codes, dtype=np.uint32)
        return np.bitwise_count(k ^ q[0][None, :]).sum(axis=1, dtype=np.int64)
    monkeypatch.setattr(oracle, "hamming", hamming)
    assert _fails(pins.test_hamming_fixture, pins.test_decode_step_uses_group_sum)


def test_merge_weight_slip_fails_a_pin(monkeypatch):
    real = oracle.lse_merge

    def lse_merge(o1, lse1, o2, lse2):
        return real(o1, lse1, o2, lse1)  # second part weighted by the first part's lse
    monkeypatch.setattr(oracle, "lse_merge", lse_merge)
    assert _fails(lambda: pins.test_lse_merge_any_partition(0), pins.test_attention_fixture_and_merge)


def test_the_unmutated_oracle_passes_the_same_pin_calls():
    assert not _fails(*_normw_pins())
    assert not _fails(pins.test_gather_pages_identity_table_is_a_reshape, pins.test_gather_pages_permuted_table,
                      pins.test_paged_retrieval_equals_contiguous_retrieval)
    assert not _fails(pins.test_topk_fixture, lambda: pins.test_topk_brute_force_rank(0), pins.test_hamming_fixture,
                      pins.test_decode_step_uses_group_sum, lambda: pins.test_lse_merge_any_partition(0),
                      pins.test_attention_fixture_and_merge)
