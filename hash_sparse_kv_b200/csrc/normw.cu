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
#include <algorithm>

#include "internal.h"
#include "normw_select.cuh"

namespace hkv {
namespace {

using namespace nw;

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

// One block per (pair, segment): block x covers pair x / nseg and the
// candidates [seg * seg_len, min((seg + 1) * seg_len, C)) of its window.
// With one segment it writes the pair's result; with several, each
// segment's own top-k (scores included, -1 / -inf padded to out_stride)
// goes to the workspace for normw_merge_kernel.
template <int W, int NP>
__global__ void __launch_bounds__(kThreads, 1) normw_kernel(NormwArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  // programmatic dependent launch: the next kernel may launch now; this
  // block reads global memory only after the previous kernel has finished
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];
  __shared__ uint32_t cnt_s[2 * kWarps];

  const int tid = threadIdx.x;
  const int p = blockIdx.x / a.nseg, seg = blockIdx.x % a.nseg;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  const int s0 = seg * a.seg_len;
  const int C = min(a.seg_len, a.C - s0);
  const int k_eff = min(a.top_k, C);
  int32_t* idx = a.idx + (int64_t)blockIdx.x * a.out_stride;
  float* score = a.score != nullptr ? a.score + (int64_t)blockIdx.x * a.out_stride : nullptr;
  for (int i = k_eff + tid; i < a.out_stride; i += kThreads) {
    idx[i] = -1;
    if (score != nullptr) score[i] = -INFINITY;
  }
  if (k_eff <= 0) return;

  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.g;
  for (int i = tid; i < a.g * W; i += kThreads) qc_s[i] = a.q_codes[qrow0 * W + i];
  __syncthreads();
  const int64_t row0 = (int64_t)p * a.cap + a.lo + s0;
  block_select<W, NP>(a.k_codes + row0 * W, a.norms + row0, a.vec_norms != 0, qc_s, a.g, a.gb, a.lo + s0, C, k_eff,
                      smem, wsum, found, cnt_s, idx, score);
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
  // programmatic dependent launch: the next kernel may launch now; this
  // block reads global memory only after the previous kernel has finished
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)P * a.nseg));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fn, a);
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
  cfg.gridDim = dim3((unsigned)P);
  cfg.dynamicSmemBytes = kRegionBytes;
  return cuda_check(cudaLaunchKernelEx(&cfg, normw_merge_kernel, m), "norm-weighted retrieval merge launch");
}

}  // namespace hkv
