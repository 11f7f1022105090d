// HashEvict eviction (HashEvict, "Abstract"): at every decoding step the new
// token's key and value replace the cached token expected to receive the
// lowest attention -- the one whose binarized projection is farthest in
// Hamming distance from the query's.  The scan reuses the group-summed
// bit-sliced distance of the retrieval kernels.
#include <algorithm>

#include "hamming.cuh"
#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 16;

int bit_length(int v) {
  int n = 0;
  while (v) {
    ++n;
    v >>= 1;
  }
  return n;
}

// Candidates [sink_end, local_start); ties to the lowest t.  Each
// block reduces its range to one 64-bit key (D << 32 | ~t) and folds it into
// the pair's slot with atomicMax; the largest key is the largest D with the
// smallest t.  A second launch turns the keys into indices and clears them.
template <int W, int NP>
__global__ void __launch_bounds__(kThreads)
evict_scan_kernel(const uint32_t* __restrict__ q_codes, const uint32_t* __restrict__ k_codes, int Hq, int Hkv, int g,
                  int64_t cap, int lo, int C, int per_block, int nseg, unsigned long long* best) {
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ unsigned long long warp_best[kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x / nseg, seg = blockIdx.x % nseg;
  const int64_t qrow0 = (int64_t)(p / Hkv) * Hq + (int64_t)(p % Hkv) * g;
  for (int i = tid; i < g * W; i += kThreads) qc_s[i] = q_codes[qrow0 * W + i];
  __syncthreads();
  Planes<W, NP> planes;
  build_planes<W, NP>(qc_s, g, planes);
  const int s0 = seg * per_block, s1 = min(s0 + per_block, C);
  unsigned long long mx = 0ull;
  const uint32_t* base = k_codes + ((int64_t)p * cap + lo) * W;
  constexpr int kU = 4;  // codes in flight per thread
  for (int t0 = s0 + tid; t0 < s1; t0 += kU * kThreads) {
    uint32_t ck[kU][W];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int t = t0 + u * kThreads;
      if (t < s1) ld_stream(base + (int64_t)t * W, ck[u]);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int t = t0 + u * kThreads;
      if (t < s1) {
        const unsigned long long key =
            ((unsigned long long)token_distance<W, NP>(ck[u], planes) << 32) | (0xFFFFFFFFu - (uint32_t)(lo + t));
        mx = key > mx ? key : mx;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const unsigned long long o = __shfl_xor_sync(0xffffffffu, mx, off);
    mx = o > mx ? o : mx;
  }
  if (lane == 0) warp_best[warp] = mx;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bm = 0ull;
    for (int w = 0; w < kWarps; ++w) bm = warp_best[w] > bm ? warp_best[w] : bm;
    if (bm != 0ull) atomicMax(best + p, bm);
  }
}

__global__ void evict_finish_kernel(unsigned long long* best, int P, int32_t* victim, int32_t* vdist) {
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
    const unsigned long long v = best[p];
    victim[p] = v ? (int32_t)(0xFFFFFFFFu - (uint32_t)v) : -1;
    if (vdist != nullptr) vdist[p] = v ? (int32_t)(v >> 32) : -1;
    best[p] = 0ull;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
write_slots_kernel(int P, int W, const T* __restrict__ k_new, const T* __restrict__ v_new,
                   const uint32_t* __restrict__ codes_new, const uint16_t* __restrict__ norms_new, T* K, T* V,
                   uint32_t* codes, uint16_t* norms, int64_t cap, const int32_t* __restrict__ slot, int32_t* status) {
  constexpr int EPC = 16 / sizeof(T), CPR = kHeadDim / EPC;  // 16-byte chunks per row
  const int per_pair = 2 * CPR + 1;                          // K chunks, V chunks, code + norm
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < P * per_pair; i += gridDim.x * blockDim.x) {
    const int p = i / per_pair, j = i % per_pair;
    const int s = slot[p];
    if (s < 0) continue;
    if (s >= cap) {
      if (j == 0) report(status, HKV_ERR_DEVICE_RANGE);
      continue;
    }
    const int64_t row = (int64_t)p * cap + s;
    if (j < CPR) {
      reinterpret_cast<uint4*>(K + row * kHeadDim)[j] = reinterpret_cast<const uint4*>(k_new + (int64_t)p * kHeadDim)[j];
    } else if (j < 2 * CPR) {
      reinterpret_cast<uint4*>(V + row * kHeadDim)[j - CPR] =
          reinterpret_cast<const uint4*>(v_new + (int64_t)p * kHeadDim)[j - CPR];
    } else {
      for (int w = 0; w < W; ++w) codes[row * W + w] = codes_new[(int64_t)p * W + w];
      if (norms != nullptr && norms_new != nullptr) norms[row] = norms_new[p];
    }
  }
}

}  // namespace

int launch_evict(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes, int32_t* victim,
                 int32_t* vdist, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0) return HKV_OK;
  if (ws == nullptr || ws_bytes < sizeof(unsigned long long) * (size_t)P)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, sizeof(unsigned long long) * (size_t)P);
  const Window w = window(s.N, s.n_sink, s.n_local);
  const int g = s.Hq / s.Hkv, np = bit_length(g);
  auto* best = static_cast<unsigned long long*>(ws);
  if (w.C > 0) {
    using EvictFn = void (*)(const uint32_t*, const uint32_t*, int, int, int, int64_t, int, int, int, int,
                             unsigned long long*);
    EvictFn fn = nullptr;
#define HKV_EV(WV, NPV) \
  if (s.words == WV && np == NPV) fn = evict_scan_kernel<WV, NPV>;
    HKV_EV(2, 1) HKV_EV(2, 2) HKV_EV(2, 3) HKV_EV(2, 4) HKV_EV(2, 5)
    HKV_EV(4, 1) HKV_EV(4, 2) HKV_EV(4, 3) HKV_EV(4, 4) HKV_EV(4, 5)
#undef HKV_EV
    if (fn == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no eviction kernel for %d-bit codes and group %d", s.words * 32, g);
    const int64_t target = 4LL * sm_count();
    int64_t nseg = std::max<int64_t>(1, std::min<int64_t>(ceil_div(w.C, 1024), ceil_div(target, P)));
    const int per_block = (int)ceil_div(w.C, nseg);
    nseg = ceil_div(w.C, per_block);
    fn<<<(unsigned)(P * nseg), kThreads, 0, st>>>(q_codes, k_codes, s.Hq, s.Hkv, g, s.cap, (int)w.sink_end,
                                                   (int)w.C, per_block, (int)nseg, best);
    int rc = cuda_check(cudaGetLastError(), "evict scan launch");
    if (rc != HKV_OK) return rc;
  }
  evict_finish_kernel<<<(unsigned)std::min<int64_t>(ceil_div(P, 256), 1024), 256, 0, st>>>(best, P, victim, vdist);
  return cuda_check(cudaGetLastError(), "evict finish launch");
}

int launch_write_slots(int dtype, int P, int W, const void* k_new, const void* v_new, const uint32_t* codes_new,
                       const uint16_t* norms_new, void* K, void* V, uint32_t* codes, uint16_t* norms, int64_t cap,
                       const int32_t* slot, int32_t* status, cudaStream_t st) {
  if (P == 0) return HKV_OK;
  const int per_pair = 2 * (dtype == HKV_BF16 ? 16 : 32) + 1;
  const int64_t total = (int64_t)P * per_pair;
  const unsigned grid = (unsigned)std::min<int64_t>(ceil_div(total, kThreads), 4LL * sm_count());
  if (dtype == HKV_BF16)
    write_slots_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
        P, W, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), codes_new, norms_new,
        static_cast<__nv_bfloat16*>(K), static_cast<__nv_bfloat16*>(V), codes, norms, cap, slot, status);
  else
    write_slots_kernel<float><<<grid, kThreads, 0, st>>>(P, W, static_cast<const float*>(k_new),
                                                         static_cast<const float*>(v_new), codes_new, norms_new,
                                                         static_cast<float*>(K), static_cast<float*>(V), codes, norms,
                                                         cap, slot, status);
  return cuda_check(cudaGetLastError(), "write slots launch");
}

}  // namespace hkv
