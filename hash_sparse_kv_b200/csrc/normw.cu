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
// One block of 512 threads per (batch, KV head) pair, candidates up to
// 65536 (their distances stay in shared memory):
//  * scan: stream the codes (16 warps, each a contiguous range), compute D
//    with the bit-sliced group distance, keep it in shared memory and count
//    the top 11 bits of each token's order key in a 2048-bin histogram;
//  * radix select: find the bin holding the k-th best key, then refine its
//    prefix by the next 11 and the last 10 bits over the tokens that share
//    it (stopping early once a whole bin is taken), which yields the exact
//    threshold key and how many of the tokens equal to it are taken;
//  * ordered compaction: every warp counts its strict and tied tokens, and
//    then writes its selected tokens at their ascending positions.
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

struct NormwArgs {
  const uint32_t* q_codes;  // [B, Hq, W]
  const uint32_t* k_codes;  // [B, Hkv, cap, W]
  const uint16_t* norms;    // [B, Hkv, cap] fp16
  int Hq, Hkv, g, gb;
  int64_t cap;
  int lo, C, k_eff, top_k;
  int range;      // tokens per warp, a multiple of kChunk
  int vec_norms;  // norms of every pair start on a 16-byte boundary
  int32_t* idx;   // [B, Hkv, top_k]
  float* score;   // nullable [B, Hkv, top_k]
};

__device__ __forceinline__ float token_score(int D, uint16_t nbits, int gb) {
  return __half2float(__ushort_as_half(nbits)) * (float)(gb - 2 * D);
}

// Larger score -> smaller key; -0 and +0 are one score.
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? u : (~u & 0x7FFFFFFFu);
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
// tokens (8 consecutive tokens per lane); all loads of a group are issued
// before its first use.  Chunks at or past t_end are skipped (warp-uniform).
constexpr int kG = 4;
struct Group {
  uint4 d[kG], n[kG];
  __device__ __forceinline__ void load(const uint16_t* dist_s, const uint16_t* nr, int base, int t_end, bool vec,
                                       int lane) {
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
};

template <int W, int NP>
__global__ void __launch_bounds__(kThreads, 1) normw_kernel(NormwArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);              // [kBins]
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(smem + kBins * 4);  // [kWarps * range]
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];
  __shared__ uint32_t cnt_s[2 * kWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  int32_t* idx = a.idx + (int64_t)p * a.top_k;
  float* score = a.score != nullptr ? a.score + (int64_t)p * a.top_k : nullptr;
  for (int i = a.k_eff + tid; i < a.top_k; i += kThreads) {
    idx[i] = -1;
    if (score != nullptr) score[i] = -INFINITY;
  }
  if (a.k_eff == 0) return;

  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.g;
  for (int i = tid; i < a.g * W; i += kThreads) qc_s[i] = a.q_codes[qrow0 * W + i];
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();

  const int64_t row0 = (int64_t)p * a.cap + a.lo;
  const uint32_t* kc = a.k_codes + row0 * W;
  const uint16_t* nr = a.norms + row0;
  const int t_beg = warp * a.range, t_end = min(t_beg + a.range, a.C);
  const bool vec = a.vec_norms != 0;

  // ---- scan: distances to shared memory, histogram of key bits [21, 32)
  {
    Planes<W, NP> planes;
    build_planes<W, NP>(qc_s, a.g, planes);
    constexpr int kU = 8;  // codes in flight per thread
    for (int base = t_beg; base < t_end; base += 32 * kU) {
      uint32_t ck[kU][W];
      uint16_t nb[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = base + u * 32 + lane;
        nb[u] = 0;
        if (t < t_end) {
          ld_stream(kc + (int64_t)t * W, ck[u]);
          nb[u] = nr[t];
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = base + u * 32 + lane;
        const bool valid = t < t_end;
        int D = 0;
        if (valid) {
          D = token_distance<W, NP>(ck[u], planes);
          dist_s[t] = (uint16_t)D;
        }
        hist_add(hist, order_key(token_score(D, nb[u], a.gb)) >> 21, valid);
      }
    }
  }
  __syncthreads();

  // ---- radix select: prefix of `bits` resolved bits, k_rem still to take
  uint32_t prefix = 0u, k_rem = (uint32_t)a.k_eff;
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
      Group gr;
      gr.load(dist_s, nr, base, t_end, vec, lane);
#pragma unroll
      for (int u = 0; u < kG; ++u) {
        if (base + u * kChunk >= t_end) break;
        const int t = base + u * kChunk + lane * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t key = order_key(token_score((int)half_at(gr.d[u], j), (uint16_t)half_at(gr.n[u], j), a.gb));
          hist_add(hist, (key >> nsh) & mask, t + j < t_end && (key >> sh) == prefix);
        }
      }
    }
    __syncthreads();
  }
  // selected: key >> sh < prefix, or key >> sh == prefix among the first
  // `need` such tokens in index order
  const uint32_t need = k_rem;

  // ---- ordered compaction
  uint32_t n_strict = 0u, n_tie = 0u;
  for (int base = t_beg; base < t_end; base += kG * kChunk) {
    Group gr;
    gr.load(dist_s, nr, base, t_end, vec, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int t = base + u * kChunk + lane * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t k =
            order_key(token_score((int)half_at(gr.d[u], j), (uint16_t)half_at(gr.n[u], j), a.gb)) >> sh;
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
    Group gr;
    gr.load(dist_s, nr, base, t_end, vec, lane);
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      if (base + u * kChunk >= t_end) break;
      const int t = base + u * kChunk + lane * 8;
      uint32_t strict_m = 0u, tie_m = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t k =
            order_key(token_score((int)half_at(gr.d[u], j), (uint16_t)half_at(gr.n[u], j), a.gb)) >> sh;
        const bool v = t + j < t_end;
        strict_m |= (v && k < prefix) ? 1u << j : 0u;
        tie_m |= (v && k == prefix) ? 1u << j : 0u;
      }
      const uint32_t lt = (uint32_t)__popc(tie_m);
      const uint32_t tie_incl = warp_incl_sum(lt, lane);
      uint32_t rank = tie_seen + tie_incl - lt;  // tie rank of this lane's first tied token
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
          idx[out] = a.lo + t + j;
          if (score != nullptr)
            score[out] = token_score((int)half_at(gr.d[u], j), (uint16_t)half_at(gr.n[u], j), a.gb);
          ++out;
        }
      pos += __shfl_sync(0xffffffffu, sel_incl, 31);
      tie_seen += __shfl_sync(0xffffffffu, tie_incl, 31);
    }
  }
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

int launch_retrieve_normw(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                          const uint16_t* norms, int32_t* idx, float* score, cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  const Window w = window(s.N, s.n_sink, s.n_local);
  if (w.C > kMaxTokens)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates per KV head (norm-weighted retrieval takes up to %d)",
                (long long)w.C, kMaxTokens);
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
  a.k_eff = (int)std::min<int64_t>(s.top_k, w.C);
  a.top_k = s.top_k;
  a.range = (int)(ceil_div(std::max<int64_t>(w.C, 1), (int64_t)kWarps * kChunk) * kChunk);
  a.vec_norms = (reinterpret_cast<uintptr_t>(norms) % 16 == 0 && s.cap % 8 == 0 && w.sink_end % 8 == 0) ? 1 : 0;
  a.idx = idx;
  a.score = score;
  using Fn = void (*)(NormwArgs);
  Fn fn = nullptr;
#define HKV_NW(WV, NPV) \
  if (s.words == WV && np == NPV) fn = normw_kernel<WV, NPV>;
  HKV_NW(2, 1) HKV_NW(2, 2) HKV_NW(2, 3) HKV_NW(2, 4) HKV_NW(2, 5)
  HKV_NW(4, 1) HKV_NW(4, 2) HKV_NW(4, 3) HKV_NW(4, 4) HKV_NW(4, 5)
#undef HKV_NW
  if (fn == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no kernel for %d-bit codes and group %d", s.words * 32, g);
  const size_t smem = (size_t)kBins * 4 + (size_t)kWarps * a.range * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "norm-weighted retrieval shared memory");
  fn<<<(unsigned)P, kThreads, smem, st>>>(a);
  return cuda_check(cudaGetLastError(), "norm-weighted retrieval launch");
}

}  // namespace hkv
