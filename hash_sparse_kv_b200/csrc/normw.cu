// Norm-weighted sign-VQ retrieval (Self-Indexing KVCache, "Abstract": the
// sign code of a key is its 1-bit vector quantisation, kept beside the key's
// norm).  Reading the stored pair as the key's reconstruction
// |k| * sign(k) / sqrt(b) and the query head as sign(q_h) / sqrt(b), their
// inner product is |k| (b - 2 popcount(cq_h XOR ck)) / b.  Summed over the g
// query heads of a KV head, the score of token t is
//     S(t) = norm_t * (g * b - 2 * D(t)),   D(t) = sum_h popcount(cq_h XOR ck_t),
// and each KV head keeps the top_k candidates with the LARGEST S, ties to
// the lowest index.  norm_t is the stored fp16 value; the product has at
// most 11 + 12 significant bits, so the fp32 score is exact.
//
// One block of 512 threads per (batch, KV head) pair and segment of at most
// 65536 candidates (one 16-bit word per candidate stays in shared memory):
//  * scan: stream the codes (16 warps, each a contiguous range), compute D
//    with the bit-sliced group distance and the score, keep the top 16 bits
//    of the score's order key in shared memory and count their top 11 bits
//    in a 2048-bin histogram;
//  * radix select: find the bin b0 holding the k-th best key; one pass over
//    the kept bits lists (per warp, in token order) every token at or below
//    b0, usually a few thousand; their full keys are computed again from
//    their codes and norms, and the next 11 and the last 10 key bits are
//    resolved over the lists only (stopping early once a whole bin is
//    taken), which yields the exact threshold key and how many of the
//    tokens equal to it are taken;
//  * ordered compaction over the lists: every warp counts its strict and
//    tied tokens, then writes its selected tokens at their ascending
//    positions.
// When the listed tokens do not fit the lists (long runs of equal scores,
// or the best tokens crowded into one warp's range) the block recomputes
// the distances into shared memory and runs the select and the compaction
// as full passes over every token instead.
// A pair with more candidates than one block holds, or with too few pairs
// to fill the GPU, is cut into segments: each segment's top-k goes to a
// workspace, and a second launch (one block per pair) selects among those
// lists in the same way.
// The order key maps a larger score to a smaller unsigned key, so "the k
// best" is "the k smallest keys".
#include <cuda_fp16.h>

#include <algorithm>

#include "hamming.cuh"
#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 16;
constexpr int kBins = 2048;  // 11-bit digits
constexpr int kChunk = 256;  // tokens per warp step in the select passes (8 per lane)
constexpr int kMaxTokens = 65536;
constexpr int kListCap = 512;  // list entries per warp in the select
constexpr size_t kRegionBytes = (size_t)2 * kWarps * kListCap * 4;  // the lists: keys, then positions

struct NormwArgs {
  const uint32_t* q_codes;  // [B, Hq, W]
  const uint32_t* k_codes;  // [B, Hkv, cap, W]
  const uint16_t* norms;    // [B, Hkv, cap] fp16
  int Hq, Hkv, g, gb;
  int64_t cap;
  int lo, C;        // the candidate window [lo, lo + C) of every pair
  int top_k;        // entries selected per block (at most its candidates)
  int nseg;         // segments per pair
  int seg_len;      // candidates per segment (a multiple of kWarps * kChunk when nseg > 1)
  int out_stride;   // output entries per block (top_k with one segment)
  int vec_norms;    // norms of every block start on a 16-byte boundary
  int32_t* idx;     // [P * nseg, out_stride]
  float* score;     // nullable [P * nseg, out_stride]
};

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
__device__ void find_bin(const uint32_t* hist, uint32_t k_rem, uint32_t* wsum, uint32_t* out) {
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

// One block per (pair, segment): block x covers pair x / nseg and the
// candidates [seg * seg_len, min((seg + 1) * seg_len, C)) of its window.
// With one segment it writes the pair's result; with several, each
// segment's own top-k (scores included, -1 / -inf padded to out_stride)
// goes to the workspace for normw_merge_kernel.
template <int W, int NP>
__global__ void __launch_bounds__(kThreads, 1) normw_kernel(NormwArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* region = reinterpret_cast<uint32_t*>(smem);                    // the select's lists
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kRegionBytes);       // [kBins]
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(smem + kRegionBytes + kBins * 4);  // [kWarps * range]
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];
  __shared__ uint32_t cnt_s[2 * kWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x / a.nseg, seg = blockIdx.x % a.nseg;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  const int s0 = seg * a.seg_len;
  const int C = min(a.seg_len, a.C - s0);
  const int k_eff = min(a.top_k, C);
  const int range = ((C + kWarps * kChunk - 1) / (kWarps * kChunk)) * kChunk;
  int32_t* idx = a.idx + (int64_t)blockIdx.x * a.out_stride;
  float* score = a.score != nullptr ? a.score + (int64_t)blockIdx.x * a.out_stride : nullptr;
  for (int i = k_eff + tid; i < a.out_stride; i += kThreads) {
    idx[i] = -1;
    if (score != nullptr) score[i] = -INFINITY;
  }
  if (k_eff <= 0) return;

  const int64_t row0 = (int64_t)p * a.cap + a.lo + s0;
  const uint32_t* kc = a.k_codes + row0 * W;
  const uint16_t* nr = a.norms + row0;

  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.g;
  for (int i = tid; i < a.g * W; i += kThreads) qc_s[i] = a.q_codes[qrow0 * W + i];
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  const int t_beg = warp * range, t_end = min(t_beg + range, C);

  // ---- scan: key bits to shared memory, histogram of their top 11 bits
  scan_range<W, NP, true>(kc, nr, qc_s, a.g, a.gb, t_beg, t_end, dist_s, hist);
  __syncthreads();

  NormSrc src;
  src.dist_s = dist_s;
  src.nr = nr;
  src.vec = a.vec_norms != 0;
  src.gb = a.gb;
  src.lo = a.lo + s0;
  uint32_t* lkey = region;
  uint32_t* lpos = region + kWarps * kListCap;
  if (select_key16<W, NP>(dist_s, kc, nr, qc_s, a.g, a.gb, src, t_beg, t_end, (uint32_t)k_eff, hist, wsum, found,
                          cnt_s, lkey, lpos, idx, score))
    return;
  // the lists overflowed: distances in place of the key bits, then full passes
  scan_range<W, NP, false>(kc, nr, qc_s, a.g, a.gb, t_beg, t_end, dist_s, hist);
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  hist_top(src, t_beg, t_end, hist, lane);
  __syncthreads();
  select_and_write(src, t_beg, t_end, (uint32_t)k_eff, hist, wsum, found, cnt_s, idx, score);
}

struct MergeArgs {
  const float* sc;    // [P, L] the segments' scores, -inf past each segment's count
  const int32_t* ci;  // [P, L] their token indices
  int L;              // entries per pair, a multiple of 8
  int range;          // entries per warp, a multiple of kChunk
  int k_eff, top_k;
  int32_t* idx;  // [P, top_k]
  float* score;  // nullable [P, top_k]
};

// One block per pair: the pair's top k_eff among its segments' selections.
// Every token of the pair's top-k is in its own segment's top-k (the order
// within a segment is the pair's order restricted to it), and the lists
// run in segment order with ascending tokens inside each, so position
// order is token order: ties to the lowest position are ties to the
// lowest token, and ascending positions give ascending tokens.  Padding
// entries score -inf, below every finite score, and k_eff is at most the
// number of real entries, so no padding entry is selected.
__global__ void __launch_bounds__(kThreads, 1) normw_merge_kernel(MergeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem);  // [2][kWarps][kListCap]
  __shared__ __align__(16) uint32_t hist[kBins];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];
  __shared__ uint32_t cnt_s[2 * kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x;
  int32_t* idx = a.idx + (int64_t)p * a.top_k;
  float* score = a.score != nullptr ? a.score + (int64_t)p * a.top_k : nullptr;
  for (int i = a.k_eff + tid; i < a.top_k; i += kThreads) {
    idx[i] = -1;
    if (score != nullptr) score[i] = -INFINITY;
  }
  if (a.k_eff <= 0) return;
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  CandSrc src;
  src.sc = a.sc + (int64_t)p * a.L;
  src.ci = a.ci + (int64_t)p * a.L;
  const int t_beg = warp * a.range, t_end = min(t_beg + a.range, a.L);
  hist_top(src, t_beg, t_end, hist, lane);
  __syncthreads();
  select_entries(src, t_beg, t_end, (uint32_t)a.k_eff, hist, wsum, found, cnt_s, lists, lists + kWarps * kListCap,
                 idx, score);
}

int bit_length(int v) {
  int n = 0;
  while (v) {
    ++n;
    v >>= 1;
  }
  return n;
}

}  // namespace

NormwPlan normw_plan(int P, int64_t C, int top_k, int sms) {
  NormwPlan pl;
  const int64_t step = (int64_t)kWarps * kChunk;
  if (P <= 0 || C <= 0 || top_k <= 0) return pl;
  const int64_t nmin = ceil_div(C, (int64_t)kMaxTokens);
  const int64_t nfill = std::max<int64_t>(1, sms / P);
  int64_t n = std::max(nmin, std::min(nfill, ceil_div(C, step)));
  if (n <= 1) return pl;
  const int64_t len = ceil_div(ceil_div(C, n), step) * step;
  n = ceil_div(C, len);
  if (n <= 1) return pl;
  pl.nseg = (int)n;
  pl.seg_len = (int)len;
  pl.stride = (int)(ceil_div(std::min<int64_t>(top_k, len), (int64_t)8) * 8);
  pl.ws_bytes = (size_t)P * (size_t)n * (size_t)pl.stride * 8u;
  return pl;
}

int launch_retrieve_normw(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                          const uint16_t* norms, int32_t* idx, float* score, void* ws, size_t ws_bytes,
                          cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  const Window w = window(s.N, s.n_sink, s.n_local);
  if (w.C > (int64_t)INT32_MAX - kMaxTokens)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates per KV head", (long long)w.C);
  NormwPlan pl;
  if (ws != nullptr) pl = normw_plan(P, w.C, s.top_k, sm_count());
  if (pl.nseg == 1 && w.C > kMaxTokens)
    return fail(HKV_ERR_UNSUPPORTED,
                "%lld candidates per KV head: above %d, norm-weighted retrieval needs a workspace",
                (long long)w.C, kMaxTokens);
  if (pl.nseg > 1 && ws_bytes < pl.ws_bytes)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, pl.ws_bytes);
  if (pl.nseg > 1 && reinterpret_cast<uintptr_t>(ws) % 16 != 0)
    return fail(HKV_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  const int g = s.Hq / s.Hkv, np = bit_length(g);
  NormwArgs a;
  a.q_codes = q_codes;
  a.k_codes = k_codes;
  a.norms = norms;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = g;
  a.gb = g * s.words * 32;
  a.cap = s.cap;
  a.lo = (int)w.sink_end;
  a.C = (int)w.C;
  a.top_k = s.top_k;
  a.nseg = pl.nseg;
  a.seg_len = pl.nseg > 1 ? pl.seg_len : (int)std::max<int64_t>(w.C, 1);
  a.vec_norms = (reinterpret_cast<uintptr_t>(norms) % 16 == 0 && s.cap % 8 == 0 && w.sink_end % 8 == 0) ? 1 : 0;
  int32_t* seg_idx = nullptr;
  float* seg_score = nullptr;
  if (pl.nseg > 1) {
    seg_idx = static_cast<int32_t*>(ws);
    seg_score = reinterpret_cast<float*>(seg_idx + (size_t)P * pl.nseg * pl.stride);
    a.out_stride = pl.stride;
    a.idx = seg_idx;
    a.score = seg_score;
  } else {
    a.out_stride = s.top_k;
    a.idx = idx;
    a.score = score;
  }
  using Fn = void (*)(NormwArgs);
  Fn fn = nullptr;
#define HKV_NW(WV, NPV) \
  if (s.words == WV && np == NPV) fn = normw_kernel<WV, NPV>;
  HKV_NW(2, 1) HKV_NW(2, 2) HKV_NW(2, 3) HKV_NW(2, 4) HKV_NW(2, 5)
  HKV_NW(4, 1) HKV_NW(4, 2) HKV_NW(4, 3) HKV_NW(4, 4) HKV_NW(4, 5)
#undef HKV_NW
  if (fn == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no kernel for %d-bit codes and group %d", s.words * 32, g);
  const int64_t range = ceil_div((int64_t)a.seg_len, (int64_t)kWarps * kChunk) * kChunk;
  const size_t smem = kRegionBytes + (size_t)kBins * 4 + (size_t)kWarps * range * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "norm-weighted retrieval shared memory");
  fn<<<(unsigned)((int64_t)P * a.nseg), kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || pl.nseg == 1) return cuda_check(e, "norm-weighted retrieval launch");

  MergeArgs m;
  m.sc = seg_score;
  m.ci = seg_idx;
  m.L = pl.nseg * pl.stride;
  m.range = (int)(ceil_div((int64_t)m.L, (int64_t)kWarps * kChunk) * kChunk);
  m.k_eff = (int)std::min<int64_t>(s.top_k, w.C);
  m.top_k = s.top_k;
  m.idx = idx;
  m.score = score;
  e = cudaFuncSetAttribute(normw_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRegionBytes);
  if (e != cudaSuccess) return cuda_check(e, "norm-weighted merge shared memory");
  normw_merge_kernel<<<(unsigned)P, kThreads, kRegionBytes, st>>>(m);
  return cuda_check(cudaGetLastError(), "norm-weighted retrieval merge launch");
}

}  // namespace hkv
