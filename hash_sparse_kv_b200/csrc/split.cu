// Token-split retrieval and attention: one long sequence's cache is cut into
// G contiguous token ranges, one per GPU (rank r holds tokens [r0_r, r1_r),
// ranks in token order).  The method's steps are unchanged -- one top-k by
// group-summed Hamming distance over all candidates, ties to the lowest
// index, exact attention over the union, log-sum-exp merge of partials
// (RetrievalAttention, "Approach") -- they only run in pieces:
//  1. every rank takes its own top-k (hkv_retrieve_topk over its range);
//     every token of the global top-k is in its own rank's top-k;
//  2. the ranks exchange those candidates (index, distance), and each finds
//     the global threshold and keeps the selected tokens of its own range
//     (split_select_kernel);
//  3. every rank attends its own rows (hkv_sparse_attend), the ranks exchange
//     the partials, and the G partials are merged (lse_merge_n_kernel).
#include <math.h>

#include <algorithm>

#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBins = 2560;  // D in [0, g * bits], g * bits <= 2048

__device__ __forceinline__ uint32_t warp_incl(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// One block per (batch, KV head) pair p.  cand_idx / cand_dist [G, P, k]:
// rank g's candidates in ascending token order, -1 past its own k_eff.  In
// the order (rank, position) the valid candidates ascend in global token
// index, so "ties to the lowest index" is "ties to the earliest candidate".
// Writes idx_out[p] = the selected candidates of rank `me` (its own local
// indices, ascending, -1 padded).
__global__ void __launch_bounds__(kThreads) split_select_kernel(const int32_t* __restrict__ cand_idx,
                                                                const int32_t* __restrict__ cand_dist, int G,
                                                                int me, int P, int k, int nbins,
                                                                int32_t* __restrict__ idx_out, int32_t* status) {
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t res[3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x;
  for (int i = tid; i < kMaxBins; i += kThreads) hist[i] = 0u;
  if (tid == 0) res[2] = 0u;
  __syncthreads();
  // histogram of every rank's distances; ties at the threshold before rank `me`
  uint32_t valid = 0u;
  for (int i = tid; i < G * k; i += kThreads) {
    const int g = i / k, j = i % k;
    const int64_t at = ((int64_t)g * P + p) * k + j;
    if (cand_idx[at] < 0) continue;
    const int D = cand_dist[at];
    if (D < 0 || D >= nbins) {
      report(status, HKV_ERR_DEVICE_RANGE);
      continue;
    }
    atomicAdd(&hist[D], 1u);
    ++valid;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) valid += __shfl_xor_sync(0xffffffffu, valid, o);
  if (lane == 0) atomicAdd(&res[2], valid);
  __syncthreads();
  const uint32_t k_eff = min((uint32_t)k, res[2]);
  int32_t* out = idx_out + (int64_t)p * k;
  if (k_eff == 0u) {
    for (int i = tid; i < k; i += kThreads) out[i] = -1;
    return;
  }
  // threshold T: the smallest D whose cumulative count reaches k_eff
  constexpr int kPer = kMaxBins / kThreads;
  uint32_t c[kPer], s = 0u;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    c[j] = hist[tid * kPer + j];
    s += c[j];
  }
  const uint32_t incl = warp_incl(s, lane);
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t cum = incl - s;
  for (int w = 0; w < warp; ++w) cum += wsum[w];
  if (cum < k_eff && cum + s >= k_eff) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (cum + c[j] >= k_eff) {
        res[0] = (uint32_t)(tid * kPer + j);
        res[1] = k_eff - cum;  // ties at T to take
        break;
      }
      cum += c[j];
    }
  }
  __syncthreads();
  const int T = (int)res[0];
  const uint32_t need = res[1];
  // ties at T among the ranks before `me`
  uint32_t before = 0u;
  for (int i = tid; i < me * k; i += kThreads) {
    const int g = i / k, j = i % k;
    const int64_t at = ((int64_t)g * P + p) * k + j;
    before += (cand_idx[at] >= 0 && cand_dist[at] == T) ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  __syncthreads();
  if (lane == 0) wsum[warp] = before;
  __syncthreads();
  uint32_t tie_seen = 0u;
  for (int w = 0; w < kWarps; ++w) tie_seen += wsum[w];
  __syncthreads();
  // ordered compaction of rank `me`'s candidates, 32 at a time per warp step
  const int64_t mine = ((int64_t)me * P + p) * k;
  uint32_t pos = 0u;
  for (int base = 0; base < k; base += kThreads) {
    const int j = base + tid;
    int32_t t = -1;
    int D = 0;
    if (j < k) {
      t = cand_idx[mine + j];
      D = cand_dist[mine + j];
    }
    const bool strict = t >= 0 && D < T, tie = t >= 0 && D == T;
    const uint32_t tie_m = __ballot_sync(0xffffffffu, tie);
    const uint32_t tie_w = (uint32_t)__popc(tie_m);
    if (lane == 0) wsum[warp] = tie_w;
    __syncthreads();
    uint32_t tie_pre = tie_seen;  // ties before this warp's lanes in this step
    for (int w = 0; w < warp; ++w) tie_pre += wsum[w];
    const bool sel = strict || (tie && tie_pre + (uint32_t)__popc(tie_m & lanemask_lt()) < need);
    const uint32_t sel_m = __ballot_sync(0xffffffffu, sel);
    uint32_t step_ties = 0u;
    for (int w = 0; w < kWarps; ++w) step_ties += wsum[w];
    __syncthreads();
    if (lane == 0) wsum[warp] = (uint32_t)__popc(sel_m);
    __syncthreads();
    uint32_t sel_pre = pos;
    uint32_t step_sel = 0u;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) sel_pre += wsum[w];
      step_sel += wsum[w];
    }
    if (sel) out[sel_pre + (uint32_t)__popc(sel_m & lanemask_lt())] = t;
    pos += step_sel;
    tie_seen += step_ties;
    __syncthreads();
  }
  for (int i = (int)pos + tid; i < k; i += kThreads) out[i] = -1;
}

// One warp per row: out = sum_g w_g o_g / sum_g w_g with w_g = exp(lse_g - M),
// M = max_g lse_g; lse_out = M + log sum_g w_g.  Rows whose partials are all
// empty (lse -inf) give out 0, lse -inf.
__global__ void lse_merge_n_kernel(int G, int64_t rows, const float* __restrict__ o, const float* __restrict__ lse,
                                   float* __restrict__ out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int g = 0; g < G; ++g) M = fmaxf(M, lse[(int64_t)g * rows + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int g = 0; g < G; ++g) {
      const float wg = expf(lse[(int64_t)g * rows + row] - M);
      const float4 v = reinterpret_cast<const float4*>(o + ((int64_t)g * rows + row) * kHeadDim)[lane];
      acc.x += wg * v.x;
      acc.y += wg * v.y;
      acc.z += wg * v.z;
      acc.w += wg * v.w;
      L += wg;
    }
    const float inv = 1.f / L;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
  }
  reinterpret_cast<float4*>(out + row * kHeadDim)[lane] = acc;
  if (lane == 0 && lse_out != nullptr) lse_out[row] = M == -INFINITY ? -INFINITY : M + logf(L);
}

}  // namespace

int launch_split_select(int G, int me, int P, int k, int nbins, const int32_t* cand_idx, const int32_t* cand_dist,
                        int32_t* idx_out, int32_t* status, cudaStream_t st) {
  if (P == 0 || k == 0) return HKV_OK;
  if (nbins > kMaxBins) return fail(HKV_ERR_UNSUPPORTED, "%d distance bins (at most %d)", nbins, kMaxBins);
  split_select_kernel<<<(unsigned)P, kThreads, 0, st>>>(cand_idx, cand_dist, G, me, P, k, nbins, idx_out, status);
  return cuda_check(cudaGetLastError(), "split select launch");
}

int launch_lse_merge_n(int G, int64_t rows, const float* o, const float* lse, float* out, float* lse_out,
                       cudaStream_t st) {
  if (rows == 0) return HKV_OK;
  const int64_t threads = rows * 32;
  lse_merge_n_kernel<<<(unsigned)ceil_div(threads, 256), 256, 0, st>>>(G, rows, o, lse, out, lse_out);
  return cuda_check(cudaGetLastError(), "merge launch");
}

}  // namespace hkv
