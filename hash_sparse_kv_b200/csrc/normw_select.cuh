// Norm-weighted sign-VQ selection of one block's candidates (Self-Indexing
// KVCache, "Abstract"), shared by the norm-weighted retrieval kernels
// (normw.cu) and the norm-weighted decode step (retrieve.cu).  The score of
// token t for a KV head with g query heads and b-bit codes is
//     S(t) = norm_t * (g * b - 2 * D(t)),   D(t) = sum_h popcount(cq_h XOR ck_t),
// largest first, ties to the lowest index.  The design (key bits kept per
// token, lists of the tokens at or below the threshold bin, full passes as
// the fallback) is described at the top of normw.cu.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "hamming.cuh"

namespace hkv {
namespace nw {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 16;
constexpr int kBins = 2048;  // 11-bit digits
constexpr int kChunk = 256;  // tokens per warp step in the select passes (8 per lane)
constexpr int kMaxTokens = 65536;
constexpr int kListCap = 512;  // list entries per warp in the select
constexpr size_t kRegionBytes = (size_t)2 * kWarps * kListCap * 4;  // the lists: keys, then positions


__device__ __forceinline__ float token_score(int D, uint16_t nbits, int gb) {
  return __half2float(__ushort_as_half(nbits)) * (float)(gb - 2 * D);
}

// Order key of a score: a larger score gives a smaller key, and -0 and +0
// are one score.  A score is an fp16 norm (finite, magnitude below 2^16)
// times an integer m with |m| <= 16 * 128 = 2^11, so a nonzero |score| lies
// in [2^-24, 2^27): its biased fp32 exponent E is in [103, 153].  Then
// c = ((E - 102) << 23) | mantissa (29 bits, 0 for a zero score) orders the
// magnitudes, r = 2^29 +- c (30 bits) orders the scores, and the key is
// (2^30 - 1 - r) << 2.  Against the plain fp32 order key this moves two
// unused exponent bits out of the top 11 bits, so the first histogram
// splits each octave of scores into 16 bins instead of 4.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  const uint32_t mag = u & 0x7FFFFFFFu;
  const uint32_t c = mag == 0u ? 0u : mag - (102u << 23);
  const uint32_t r = (u >> 31) ? (1u << 29) - c : (1u << 29) + c;
  return ((1u << 30) - 1u - r) << 2;
}

// The score of a key (score_key inverted; a zero score comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key) {
  const uint32_t r = (1u << 30) - 1u - (key >> 2);
  const bool neg = r < (1u << 29);
  const uint32_t c = neg ? (1u << 29) - r : r - (1u << 29);
  return __uint_as_float((neg ? 0x80000000u : 0u) | (c == 0u ? 0u : c + (102u << 23)));
}

// Adds one to hist[bin] for every lane with `on` (shared-memory atomics;
// aggregating equal bins with __match_any_sync first measured slower).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool on) {
  if (on) atomicAdd(&hist[bin], 1u);
}

__device__ __forceinline__ uint32_t warp_incl_sum(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Block-wide: the bin b whose cumulative count first reaches k_rem (>= 1 and
// at most the histogram's total).  out[0] = b, out[1] = count below b,
// out[2] = count in b.  Each thread owns 4 consecutive bins.
__device__ inline void find_bin(const uint32_t* hist, uint32_t k_rem, uint32_t* wsum, uint32_t* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4 c = reinterpret_cast<const uint4*>(hist)[tid];
  const uint32_t s = c.x + c.y + c.z + c.w;
  const uint32_t incl = warp_incl_sum(s, lane);
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t excl = incl - s;
  for (int w = 0; w < warp; ++w) excl += wsum[w];
  if (excl < k_rem && excl + s >= k_rem) {
    const uint32_t v[4] = {c.x, c.y, c.z, c.w};
    uint32_t cum = excl;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (cum + v[j] >= k_rem) {
        out[0] = (uint32_t)(tid * 4 + j);
        out[1] = cum;
        out[2] = v[j];
        break;
      }
      cum += v[j];
    }
  }
}

// Eight consecutive norms of tokens [t, t + 8), packed two per word (zero
// past t_end).
__device__ __forceinline__ uint4 load_norms8(const uint16_t* nr, int t, int t_end, bool vec) {
  if (vec && t + 8 <= t_end) return *reinterpret_cast<const uint4*>(nr + t);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (t + j < t_end) w[j >> 1] |= (uint32_t)nr[t + j] << (16 * (j & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Element j (0..7) of eight packed 16-bit values.
__device__ __forceinline__ uint32_t half_at(const uint4& v, int j) {
  const uint32_t w = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
  return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
}

// The select passes walk a warp's range in groups of kG chunks of kChunk
// entries (8 consecutive entries per lane); all loads of a group are issued
// before its first use.  Chunks at or past t_end are skipped (warp-uniform).
// A source holds one group in registers and yields each entry's score and
// token index.
constexpr int kG = 4;

// The scan's entries: distances in shared memory, norms in global memory,
// entry t is token lo + t.
struct NormSrc {
  const uint16_t* dist_s;
  const uint16_t* nr;
  bool vec;
  int gb, lo;
  uint4 d[kG], n[kG];
  __device__ __forceinline__ void load(int base, int t_end, int lane) {
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int t = base + u * kChunk + lane * 8;
      d[u] = n[u] = make_uint4(0u, 0u, 0u, 0u);
      if (base + u * kChunk < t_end) {
        d[u] = *reinterpret_cast<const uint4*>(dist_s + t);
        n[u] = load_norms8(nr, t, t_end, vec);
      }
    }
  }
  __device__ __forceinline__ float score(int u, int j) const {
    return token_score((int)half_at(d[u], j), (uint16_t)half_at(n[u], j), gb);
  }
  __device__ __forceinline__ uint32_t key(int u, int j) const { return score_key(score(u, j)); }
  __device__ __forceinline__ int32_t token(int t) const { return lo + t; }
};

// The merge's entries: the segments' selected scores and token indices in
// the workspace.  Entries come in runs of 8 that are all below t_end or all
// at or past it (the lists have a multiple of 8 entries).  Padding scores
// -inf, outside the range of score_key: it gets the largest key.
struct CandSrc {
  const float* sc;
  const int32_t* ci;
  float4 s[kG][2];
  __device__ __forceinline__ void load(int base, int t_end, int lane) {
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int t = base + u * kChunk + lane * 8;
      s[u][0] = s[u][1] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (t < t_end) {
        s[u][0] = __ldcg(reinterpret_cast<const float4*>(sc + t));
        s[u][1] = __ldcg(reinterpret_cast<const float4*>(sc + t + 4));
      }
    }
  }
  __device__ __forceinline__ float score(int u, int j) const {
    const float4& v = s[u][j >> 2];
    const int c = j & 3;
    return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
  }
  // padding (-inf) after every real entry
  __device__ __forceinline__ uint32_t key(int u, int j) const {
    const float x = score(u, j);
    return x == -INFINITY ? 0xFFFFFFFFu : score_key(x);
  }
  __device__ __forceinline__ int32_t token(int t) const { return __ldcg(ci + t); }
};

// Histogram of the order keys' top 11 bits over every warp's entries.
template <class Src>
__device__ __forceinline__ void hist_top(Src& src, int t_beg, int t_end, uint32_t* hist, int lane) {
  for (int base = t_beg; base < t_end; base += kG * kChunk) {
    src.load(base, t_end, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      if (base + u * kChunk >= t_end) break;
      const int t = base + u * kChunk + lane * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) hist_add(hist, src.key(u, j) >> 21, t + j < t_end);
    }
  }
}

// Given the histogram of the top 11 key bits over the block's entries (each
// warp owns [t_beg, t_end)), selects the k_eff entries with the smallest
// order keys, ties to the lowest position, and writes their tokens (and
// scores) at idx[0..k_eff) in ascending position.
template <class Src>
__device__ __forceinline__ void select_and_write(Src& src, int t_beg, int t_end, uint32_t k_eff, uint32_t* hist,
                                                 uint32_t* wsum, uint32_t* found, uint32_t* cnt_s, int32_t* idx,
                                                 float* score) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- radix select: prefix of the resolved bits, k_rem still to take
  uint32_t prefix = 0u, k_rem = k_eff;
  int sh = 21;
  for (int pass = 0;; ++pass) {
    find_bin(hist, k_rem, wsum, found);
    __syncthreads();
    const uint32_t bin = found[0], less = found[1], cnt = found[2];
    k_rem -= less;
    prefix = pass == 0 ? bin : (prefix << (pass == 1 ? 11 : 10)) | bin;
    if (pass > 0) sh = pass == 1 ? 10 : 0;
    if (k_rem == cnt || sh == 0) break;  // the whole bin is taken, or the key is exact
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    __syncthreads();
    const int nsh = sh == 21 ? 10 : 0;
    const uint32_t mask = sh == 21 ? 0x7FFu : 0x3FFu;
    for (int base = t_beg; base < t_end; base += kG * kChunk) {
      src.load(base, t_end, lane);
#pragma unroll
      for (int u = 0; u < kG; ++u) {
        if (base + u * kChunk >= t_end) break;
        const int t = base + u * kChunk + lane * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t key = src.key(u, j);
          hist_add(hist, (key >> nsh) & mask, t + j < t_end && (key >> sh) == prefix);
        }
      }
    }
    __syncthreads();
  }
  // selected: key >> sh < prefix, or key >> sh == prefix among the first
  // `need` such entries in position order
  const uint32_t need = k_rem;

  // ---- ordered compaction
  uint32_t n_strict = 0u, n_tie = 0u;
  for (int base = t_beg; base < t_end; base += kG * kChunk) {
    src.load(base, t_end, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int t = base + u * kChunk + lane * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t k = src.key(u, j) >> sh;
        const bool v = t + j < t_end;
        n_strict += (v && k < prefix) ? 1u : 0u;
        n_tie += (v && k == prefix) ? 1u : 0u;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_strict += __shfl_xor_sync(0xffffffffu, n_strict, o);
    n_tie += __shfl_xor_sync(0xffffffffu, n_tie, o);
  }
  if (lane == 0) {
    cnt_s[warp] = n_strict;
    cnt_s[kWarps + warp] = n_tie;
  }
  __syncthreads();
  uint32_t strict_before = 0u, tie_seen = 0u;
  for (int w = 0; w < warp; ++w) {
    strict_before += cnt_s[w];
    tie_seen += cnt_s[kWarps + w];
  }
  uint32_t pos = strict_before + min(tie_seen, need);
  for (int base = t_beg; base < t_end; base += kG * kChunk) {
    src.load(base, t_end, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      if (base + u * kChunk >= t_end) break;
      const int t = base + u * kChunk + lane * 8;
      uint32_t strict_m = 0u, tie_m = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t k = src.key(u, j) >> sh;
        const bool v = t + j < t_end;
        strict_m |= (v && k < prefix) ? 1u << j : 0u;
        tie_m |= (v && k == prefix) ? 1u << j : 0u;
      }
      const uint32_t lt = (uint32_t)__popc(tie_m);
      const uint32_t tie_incl = warp_incl_sum(lt, lane);
      uint32_t rank = tie_seen + tie_incl - lt;  // tie rank of this lane's first tied entry
      uint32_t sel_m = strict_m;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (tie_m & (1u << j)) {
          if (rank < need) sel_m |= 1u << j;
          ++rank;
        }
      const uint32_t ls = (uint32_t)__popc(sel_m);
      const uint32_t sel_incl = warp_incl_sum(ls, lane);
      uint32_t out = pos + sel_incl - ls;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (sel_m & (1u << j)) {
          idx[out] = src.token(t + j);
          if (score != nullptr) score[out] = src.score(u, j);
          ++out;
        }
      pos += __shfl_sync(0xffffffffu, sel_incl, 31);
      tie_seen += __shfl_sync(0xffffffffu, tie_incl, 31);
    }
  }
}

// Finishes a select from per-warp lists holding, in ascending position,
// every entry whose key's top 11 bits are at most b0 (n entries in this
// warp's list: keys mk, positions mp).  k_rem of the entries are still to be
// taken among those in bin b0; when refine (fewer than all of them) hist
// holds bits [10, 21) of their keys.  The caller has synchronised the block after
// writing the lists and hist.
template <class Src>
__device__ __forceinline__ void list_finish(const Src& src, uint32_t b0, uint32_t k_rem, bool refine,
                                            uint32_t n, const uint32_t* mk, const uint32_t* mp, uint32_t* hist,
                                            uint32_t* wsum, uint32_t* found, uint32_t* cnt_s, int32_t* idx,
                                            float* score) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- refinement over the lists
  uint32_t prefix = b0;
  int sh = 21;
  if (refine) {
    find_bin(hist, k_rem, wsum, found);
    __syncthreads();
    k_rem -= found[1];
    const uint32_t cnt1 = found[2];
    prefix = (b0 << 11) | found[0];
    sh = 10;
    if (k_rem != cnt1) {
      for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
      __syncthreads();
      for (uint32_t i = lane; i < n; i += 32) {
        const uint32_t key = mk[i];
        hist_add(hist, key & 0x3FFu, (key >> 10) == prefix);
      }
      __syncthreads();
      find_bin(hist, k_rem, wsum, found);
      __syncthreads();
      k_rem -= found[1];
      prefix = (prefix << 10) | found[0];
      sh = 0;
    }
  }
  const uint32_t need = k_rem;

  // ---- ordered compaction over the lists
  uint32_t n_strict = 0u, n_tie = 0u;
  for (uint32_t i = lane; i < n; i += 32) {
    const uint32_t k = mk[i] >> sh;
    n_strict += k < prefix ? 1u : 0u;
    n_tie += k == prefix ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_strict += __shfl_xor_sync(0xffffffffu, n_strict, o);
    n_tie += __shfl_xor_sync(0xffffffffu, n_tie, o);
  }
  __syncthreads();  // every warp has read the overflow flags
  if (lane == 0) {
    cnt_s[warp] = n_strict;
    cnt_s[kWarps + warp] = n_tie;
  }
  __syncthreads();
  uint32_t strict_before = 0u, tie_seen = 0u;
  for (int w = 0; w < warp; ++w) {
    strict_before += cnt_s[w];
    tie_seen += cnt_s[kWarps + w];
  }
  uint32_t pos = strict_before + min(tie_seen, need);
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (uint32_t i0 = 0; i0 < n; i0 += 32) {
    const uint32_t i = i0 + lane;
    const bool v = i < n;
    const uint32_t key = v ? mk[i] : 0u;
    const uint32_t k = key >> sh;
    const bool is_tie = v && k == prefix;
    const uint32_t tie_b = __ballot_sync(0xffffffffu, is_tie);
    const bool sel = (v && k < prefix) || (is_tie && tie_seen + (uint32_t)__popc(tie_b & lt_mask) < need);
    const uint32_t sel_b = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const uint32_t o = pos + (uint32_t)__popc(sel_b & lt_mask);
      idx[o] = src.token((int)mp[i]);
      if (score != nullptr) score[o] = key_score(key);
    }
    pos += (uint32_t)__popc(sel_b);
    tie_seen += (uint32_t)__popc(tie_b);
  }
}

// The select of select_and_write with one pass over every entry.  The
// histogram of the top 11 key bits gives the bin b0 holding the k-th
// smallest key and the number of entries at or below it.  When those fit
// the warps' lists, one pass over the entries appends each one at or below
// b0 (key and position, in ascending position per warp) and counts the next
// 11 bits of those in b0; the last refinement and the ordered compaction
// then walk the lists only.  Returns false, with nothing written, when the
// entries at or below b0 do not fit (too many, or one warp's share above
// kListCap); the histogram then no longer holds the top 11 bits.
template <class Src>
__device__ __forceinline__ bool select_list(Src& src, int t_beg, int t_end, uint32_t k_eff, uint32_t* hist,
                                            uint32_t* wsum, uint32_t* found, uint32_t* cnt_s, uint32_t* lkey,
                                            uint32_t* lpos, int32_t* idx, float* score) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  find_bin(hist, k_eff, wsum, found);
  __syncthreads();
  const uint32_t b0 = found[0], less0 = found[1], cnt0 = found[2];
  if (less0 + cnt0 > (uint32_t)(kWarps * kListCap)) return false;
  uint32_t k_rem = k_eff - less0;
  const bool refine = k_rem != cnt0;
  if (refine)
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();

  // ---- the pass over every entry: lists, and bits [10, 21) of the keys in b0
  uint32_t* mk = lkey + warp * kListCap;
  uint32_t* mp = lpos + warp * kListCap;
  uint32_t n = 0u;
  bool ovf = false;
  for (int base = t_beg; base < t_end; base += kG * kChunk) {
    src.load(base, t_end, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      if (base + u * kChunk >= t_end) break;
      const int t = base + u * kChunk + lane * 8;
      uint32_t keys[8], m = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        keys[j] = src.key(u, j);
        const bool v = t + j < t_end;
        const uint32_t h = keys[j] >> 21;
        m |= (v && h <= b0) ? 1u << j : 0u;
        if (refine) hist_add(hist, (keys[j] >> 10) & 0x7FFu, v && h == b0);
      }
      const uint32_t c = (uint32_t)__popc(m);
      const uint32_t incl = warp_incl_sum(c, lane);
      const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
      if (n + tot <= (uint32_t)kListCap) {
        uint32_t o = n + incl - c;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (m & (1u << j)) {
            mk[o] = keys[j];
            mp[o] = (uint32_t)(t + j);
            ++o;
          }
        n += tot;
      } else {
        ovf = true;
      }
    }
  }
  if (lane == 0) cnt_s[warp] = ovf ? 1u : 0u;
  __syncthreads();
  bool any_ovf = false;
  for (int w = 0; w < kWarps; ++w) any_ovf |= cnt_s[w] != 0u;
  if (any_ovf) return false;

  list_finish(src, b0, k_rem, refine, n, mk, mp, hist, wsum, found, cnt_s, idx, score);
  return true;
}

// Top k_eff of the block's entries: select_list, else (the entries at or
// below the threshold bin overflow the lists) the histogram is rebuilt and
// select_and_write makes full passes.
template <class Src>
__device__ __forceinline__ void select_entries(Src& src, int t_beg, int t_end, uint32_t k_eff, uint32_t* hist,
                                               uint32_t* wsum, uint32_t* found, uint32_t* cnt_s, uint32_t* lkey,
                                               uint32_t* lpos, int32_t* idx, float* score) {
  if (select_list(src, t_beg, t_end, k_eff, hist, wsum, found, cnt_s, lkey, lpos, idx, score)) return;
  for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  hist_top(src, t_beg, t_end, hist, threadIdx.x & 31);
  __syncthreads();
  select_and_write(src, t_beg, t_end, k_eff, hist, wsum, found, cnt_s, idx, score);
}

// The scan of a block's range: each warp streams its own tokens with kU
// codes in flight per lane.  KEYS: keep the top 16 bits of each token's key
// in slot[t] and count their top 11 bits in hist; else keep the distance
// D in slot[t].  (A cp.async ring with one or two tokens per step measured
// slower: the scan is bound by the integer pipe, and the batch gives it
// independent work.)
template <int W, int NP, bool KEYS>
__device__ __forceinline__ void scan_range(const uint32_t* kc, const uint16_t* nr, const uint32_t* qc_s, int g,
                                           int gb, int t_beg, int t_end, uint16_t* slot, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  Planes<W, NP> planes;
  build_planes<W, NP>(qc_s, g, planes);
  constexpr int kU = 8;
  for (int base = t_beg; base < t_end; base += 32 * kU) {
    uint32_t ck[kU][W];
    uint16_t nb[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int t = base + u * 32 + lane;
      nb[u] = 0;
      if (t < t_end) {
        ld_stream(kc + (int64_t)t * W, ck[u]);
        if (KEYS) nb[u] = nr[t];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int t = base + u * 32 + lane;
      if (t < t_end) {
        const int D = token_distance<W, NP>(ck[u], planes);
        if (KEYS) {
          const uint32_t key = score_key(token_score(D, nb[u], gb));
          slot[t] = (uint16_t)(key >> 16);
          hist_add(hist, key >> 21, true);
        } else {
          slot[t] = (uint16_t)D;
        }
      }
    }
  }
}

// select_list for the norm-weighted scan, which kept each token's top 16
// key bits (key16): the pass over every token compares those with b0 and
// lists positions only; the listed tokens' full keys then come from their
// codes and norms again (a few thousand tokens against the range's tens of
// thousands).  Returns false, with nothing written, as select_list does.
template <int W, int NP>
__device__ __forceinline__ bool select_key16(const uint16_t* key16, const uint32_t* kc, const uint16_t* nr,
                                             const uint32_t* qc_s, int g, int gb, const NormSrc& src, int t_beg,
                                             int t_end, uint32_t k_eff, uint32_t* hist, uint32_t* wsum,
                                             uint32_t* found, uint32_t* cnt_s, uint32_t* lkey, uint32_t* lpos,
                                             int32_t* idx, float* score) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  find_bin(hist, k_eff, wsum, found);
  __syncthreads();
  const uint32_t b0 = found[0], less0 = found[1], cnt0 = found[2];
  if (less0 + cnt0 > (uint32_t)(kWarps * kListCap)) return false;
  const uint32_t k_rem = k_eff - less0;
  const bool refine = k_rem != cnt0;
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;

  // ---- the pass over every token: positions at or below b0
  uint32_t* mk = lkey + warp * kListCap;
  uint32_t* mp = lpos + warp * kListCap;
  uint32_t n = 0u;
  bool ovf = false;
  for (int base = t_beg; base < t_end; base += kChunk) {
    const int t = base + lane * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(key16 + t);
    uint32_t m = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) m |= (t + j < t_end && (half_at(v, j) >> 5) <= b0) ? 1u << j : 0u;
    const uint32_t c = (uint32_t)__popc(m);
    const uint32_t incl = warp_incl_sum(c, lane);
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    if (n + tot <= (uint32_t)kListCap) {
      uint32_t o = n + incl - c;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (m & (1u << j)) mp[o++] = (uint32_t)(t + j);
      n += tot;
    } else {
      ovf = true;
    }
  }
  if (lane == 0) cnt_s[warp] = ovf ? 1u : 0u;
  __syncthreads();
  bool any_ovf = false;
  for (int w = 0; w < kWarps; ++w) any_ovf |= cnt_s[w] != 0u;
  if (any_ovf) return false;

  // ---- full keys of the listed tokens; bits [10, 21) of those in b0
  {
    Planes<W, NP> planes;
    build_planes<W, NP>(qc_s, g, planes);
    for (uint32_t i = lane; i < n; i += 32) {
      const int t = (int)mp[i];
      uint32_t ck[W];
      ld_stream(kc + (int64_t)t * W, ck);
      const uint32_t key = score_key(token_score(token_distance<W, NP>(ck, planes), nr[t], gb));
      mk[i] = key;
      if (refine) hist_add(hist, (key >> 10) & 0x7FFu, (key >> 21) == b0);
    }
  }
  __syncthreads();
  list_finish(src, b0, k_rem, refine, n, mk, mp, hist, wsum, found, cnt_s, idx, score);
  return true;
}

// The norm-weighted top-k of one block: candidates [0, C) of the block
// (token lo + t; codes kc[t], norms nr[t]), the group's query codes in qc_s
// (complete: the caller synchronised the block after writing them).  Writes
// idx[0, k_eff) (ascending tokens) and score[0, k_eff) (nullable).  smem:
// kRegionBytes of lists, then kBins histogram words, then kWarps * range
// 16-bit words (range: C / kWarps rounded up to a multiple of kChunk).  vec: every norm row starts on a 16-byte boundary.  All threads
// call it; it ends without a final barrier.
template <int W, int NP>
__device__ __forceinline__ void block_select(const uint32_t* kc, const uint16_t* nr, bool vec, const uint32_t* qc_s,
                                             int g, int gb, int lo, int C, int k_eff, unsigned char* smem,
                                             uint32_t* wsum, uint32_t* found, uint32_t* cnt_s, int32_t* idx,
                                             float* score) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* region = reinterpret_cast<uint32_t*>(smem);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kRegionBytes);
  uint16_t* key16 = reinterpret_cast<uint16_t*>(smem + kRegionBytes + kBins * 4);
  const int range = ((C + kWarps * kChunk - 1) / (kWarps * kChunk)) * kChunk;
  const int t_beg = warp * range, t_end = min(t_beg + range, C);
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  // ---- scan: key bits to shared memory, histogram of their top 11 bits
  scan_range<W, NP, true>(kc, nr, qc_s, g, gb, t_beg, t_end, key16, hist);
  __syncthreads();
  NormSrc src;
  src.dist_s = key16;
  src.nr = nr;
  src.vec = vec;
  src.gb = gb;
  src.lo = lo;
  if (select_key16<W, NP>(key16, kc, nr, qc_s, g, gb, src, t_beg, t_end, (uint32_t)k_eff, hist, wsum, found, cnt_s,
                          region, region + kWarps * kListCap, idx, score))
    return;
  // the lists overflowed: distances in place of the key bits, then full passes
  scan_range<W, NP, false>(kc, nr, qc_s, g, gb, t_beg, t_end, key16, hist);
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  hist_top(src, t_beg, t_end, hist, lane);
  __syncthreads();
  select_and_write(src, t_beg, t_end, (uint32_t)k_eff, hist, wsum, found, cnt_s, idx, score);
}

}  // namespace nw
}  // namespace hkv
