// Retrieval over a paged cache.  The cache of every sequence is cut into
// pages of page_size tokens that live anywhere in one pool:
//     codes_pool [num_pages, Hkv, page_size, W],
// and page_table[b, j] names the pool page holding tokens
// [j * page_size, (j + 1) * page_size) of sequence b.  The method is the
// default retrieval (HashEvict, "Abstract": group-summed Hamming distance to
// the binarized query; Spotlight Attention, "Approach": keep the top-k,
// here ties to the lowest index); only the addressing differs.
//
// One block of 512 threads per (batch, KV head) pair, up to 65536
// candidates (their distances stay in shared memory):
//  * scan: each warp streams a contiguous range of tokens, looking up each
//    token's page, computes D with the bit-sliced group distance, keeps it in
//    shared memory and counts it in a histogram over [0, g * bits];
//  * the threshold T is the smallest D whose cumulative count reaches k_eff;
//  * ordered compaction: every warp counts its tokens with D < T and D == T,
//    then writes the selected ones (D < T, and D == T up to the quota in
//    index order) at their ascending positions.
// A page id outside [0, num_pages) is reported as HKV_ERR_DEVICE_RANGE and
// its tokens get the largest distance, g * bits.
#include <algorithm>

#include "hamming.cuh"
#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 16;
constexpr int kMaxBins = 2560;  // D in [0, g * bits], g * bits <= 2048
constexpr int kPerThread = kMaxBins / kThreads;
constexpr int kChunk = 256;  // tokens per warp step in the compaction (8 per lane)
constexpr int kMaxTokens = 65536;

struct PagedArgs {
  const uint32_t* q_codes;  // [B, Hq, W]
  const uint32_t* codes;    // [num_pages, Hkv, page_size, W]
  const int32_t* table;     // [B, max_pages]
  int64_t max_pages, num_pages;
  int page_size;
  int Hq, Hkv, g, dmax;  // dmax = g * bits
  int lo, C, k_eff, top_k;
  int range;      // tokens per warp, a multiple of kChunk
  int32_t* idx;   // [B, Hkv, top_k]
  int32_t* dist;  // nullable [B, Hkv, top_k]
  int32_t* status;
};

__device__ __forceinline__ uint32_t warp_incl(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

template <int W, int NP>
__global__ void __launch_bounds__(kThreads, 1) paged_topk_kernel(PagedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(smem);  // [kWarps * range]
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t cnt_s[2 * kWarps];
  __shared__ uint32_t res[2];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  int32_t* idx = a.idx + (int64_t)p * a.top_k;
  int32_t* dist = a.dist != nullptr ? a.dist + (int64_t)p * a.top_k : nullptr;
  for (int i = a.k_eff + tid; i < a.top_k; i += kThreads) {
    idx[i] = -1;
    if (dist != nullptr) dist[i] = -1;
  }
  if (a.k_eff == 0) return;

  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.g;
  for (int i = tid; i < a.g * W; i += kThreads) qc_s[i] = a.q_codes[qrow0 * W + i];
  for (int i = tid; i < kMaxBins; i += kThreads) hist[i] = 0u;
  __syncthreads();

  const int32_t* table = a.table + (int64_t)b * a.max_pages;
  const int t_beg = warp * a.range, t_end = min(t_beg + a.range, a.C);

  // ---- scan: distances to shared memory, histogram of D
  {
    Planes<W, NP> planes;
    build_planes<W, NP>(qc_s, a.g, planes);
    constexpr int kU = 8;  // codes in flight per thread
    for (int base = t_beg; base < t_end; base += 32 * kU) {
      uint32_t ck[kU][W];
      bool ok[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = base + u * 32 + lane;
        ok[u] = false;
        if (t < t_end) {
          const int tok = a.lo + t;
          const int pg = table[tok / a.page_size];
          if (pg >= 0 && pg < a.num_pages) {
            ok[u] = true;
            ld_stream(a.codes + (((int64_t)pg * a.Hkv + kvh) * a.page_size + tok % a.page_size) * W, ck[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int t = base + u * 32 + lane;
        if (t < t_end) {
          int D = a.dmax;
          if (ok[u]) {
            D = token_distance<W, NP>(ck[u], planes);
          } else {
            report(a.status, HKV_ERR_DEVICE_RANGE);
          }
          dist_s[t] = (uint16_t)D;
          atomicAdd(&hist[D], 1u);
        }
      }
    }
  }
  __syncthreads();

  // ---- threshold: T = smallest D with cumulative count >= k_eff
  {
    uint32_t c[kPerThread], s = 0u;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      c[j] = hist[tid * kPerThread + j];
      s += c[j];
    }
    const uint32_t incl = warp_incl(s, lane);
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t cum = incl - s;
    for (int w = 0; w < warp; ++w) cum += wsum[w];
    const uint32_t k_eff = (uint32_t)a.k_eff;
    if (cum < k_eff && cum + s >= k_eff) {
#pragma unroll
      for (int j = 0; j < kPerThread; ++j) {
        if (cum + c[j] >= k_eff) {
          res[0] = (uint32_t)(tid * kPerThread + j);
          res[1] = k_eff - cum;  // ties at T to take
          break;
        }
        cum += c[j];
      }
    }
  }
  __syncthreads();
  const int T = (int)res[0];
  const uint32_t need = res[1];

  // ---- ordered compaction: counts per warp, then positions
  uint32_t n_strict = 0u, n_tie = 0u;
  for (int base = t_beg; base < t_end; base += kChunk) {
    const int t = base + lane * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(dist_s + t);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int D = (int)((w4[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
      const bool in = t + j < t_end;
      n_strict += (in && D < T) ? 1u : 0u;
      n_tie += (in && D == T) ? 1u : 0u;
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
  for (int base = t_beg; base < t_end; base += kChunk) {
    const int t = base + lane * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(dist_s + t);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t strict_m = 0u, tie_m = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int D = (int)((w4[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
      const bool in = t + j < t_end;
      strict_m |= (in && D < T) ? 1u << j : 0u;
      tie_m |= (in && D == T) ? 1u << j : 0u;
    }
    const uint32_t lt = (uint32_t)__popc(tie_m);
    const uint32_t tie_incl = warp_incl(lt, lane);
    uint32_t rank = tie_seen + tie_incl - lt;  // tie rank of this lane's first tied token
    uint32_t sel_m = strict_m;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (tie_m & (1u << j)) {
        if (rank < need) sel_m |= 1u << j;
        ++rank;
      }
    const uint32_t ls = (uint32_t)__popc(sel_m);
    const uint32_t sel_incl = warp_incl(ls, lane);
    uint32_t out = pos + sel_incl - ls;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (sel_m & (1u << j)) {
        idx[out] = a.lo + t + j;
        if (dist != nullptr) dist[out] = (int32_t)((w4[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
        ++out;
      }
    pos += __shfl_sync(0xffffffffu, sel_incl, 31);
    tie_seen += __shfl_sync(0xffffffffu, tie_incl, 31);
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

int launch_retrieve_paged(const RetrieveShape& s, const PageMap& pm, const uint32_t* q_codes,
                          const uint32_t* codes_pool, int32_t* idx, int32_t* dist, int32_t* status, cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  const Window w = window(s.N, s.n_sink, s.n_local);
  if (w.C > kMaxTokens)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates per KV head (paged retrieval takes up to %d)",
                (long long)w.C, kMaxTokens);
  const int g = s.Hq / s.Hkv, np = bit_length(g);
  PagedArgs a;
  a.q_codes = q_codes;
  a.codes = codes_pool;
  a.table = pm.table;
  a.max_pages = pm.max_pages;
  a.num_pages = pm.num_pages;
  a.page_size = pm.page_size;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = g;
  a.dmax = g * s.words * 32;
  a.lo = (int)w.sink_end;
  a.C = (int)w.C;
  a.k_eff = (int)std::min<int64_t>(s.top_k, w.C);
  a.top_k = s.top_k;
  a.range = (int)(ceil_div(std::max<int64_t>(w.C, 1), (int64_t)kWarps * kChunk) * kChunk);
  a.idx = idx;
  a.dist = dist;
  a.status = status;
  using Fn = void (*)(PagedArgs);
  Fn fn = nullptr;
#define HKV_PG(WV, NPV) \
  if (s.words == WV && np == NPV) fn = paged_topk_kernel<WV, NPV>;
  HKV_PG(2, 1) HKV_PG(2, 2) HKV_PG(2, 3) HKV_PG(2, 4) HKV_PG(2, 5)
  HKV_PG(4, 1) HKV_PG(4, 2) HKV_PG(4, 3) HKV_PG(4, 4) HKV_PG(4, 5)
#undef HKV_PG
  if (fn == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no kernel for %d-bit codes and group %d", s.words * 32, g);
  const size_t smem = (size_t)kWarps * a.range * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "paged retrieval shared memory");
  fn<<<(unsigned)P, kThreads, smem, st>>>(a);
  return cuda_check(cudaGetLastError(), "paged retrieval launch");
}

}  // namespace hkv
