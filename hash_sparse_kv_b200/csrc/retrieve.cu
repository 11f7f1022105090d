// Hamming scan + top-k selection (S4, S5).
//
// HashEvict ("Abstract") scores cached keys by the Hamming distance between
// binarized projections of the query and of each key; Spotlight Attention
// ("Approach", "Key results") keeps the top-k keys per decode step.  With
// grouped-query attention a KV head's score of token t is the sum over its g
// query heads:  D(t) = sum_h popcount(cq_h XOR ck_t)  in [0, g * bits].
//
// Design (one cooperative launch):
//  * The candidate tokens of all (batch, KV head) pairs are laid end to end
//    and cut into equal contiguous ranges, one per block, so every SM gets the
//    same number of code bytes whatever the batch shape.  A block's range
//    covers one or more "segments" (its part of one pair).
//  * Phase A, per segment: stream the codes once (16-byte loads that skip
//    L1), compute D for each token, keep D in shared memory (uint16), and
//    build the segment's histogram of D in shared memory.  Publish the
//    segment's cumulative histogram and add its counts into the pair's global
//    histogram.  Then arrive at the pair's barrier.
//  * Phase B, per segment: wait (bounded) until every segment of the pair has
//    arrived; read the pair's histogram and find the threshold T: the
//    smallest D whose cumulative count reaches k_eff.  Tokens with D < T are
//    all selected; tokens with D == T are admitted in ascending token order
//    until k_eff is reached.  From the lower segments' cumulative histograms a
//    block knows how many selected tokens precede its segment, so it writes
//    its selected tokens straight to their final, ascending positions.
//  * The last block to leave a pair zeroes the pair's global scratch, so the
//    workspace is clean for the next call.
//
// The group-summed distance is computed with bit-sliced arithmetic instead of
// g * W popcounts.  For bit position j let c_j = #{h : bit j of cq_h is 1}.
// The contribution of position j is (ck_j ? g - c_j : c_j).  The NP bit planes
// of c_j (C planes) and of g - c_j (U planes) are built once per segment; per
// token each word gives NP planes V_b = (ck & U_b) | (~ck & C_b), the words'
// planes are added with carry-save adders, and D = sum_b 2^b popcount(S_b).
#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;
constexpr int kMaxTokensPerBlock = 24576;  // uint16 distances kept in shared memory
constexpr int kMinTokensPerBlock = 1024;
constexpr int kMaxBlocksPerSM = 3;

struct RetrieveArgs {
  const uint32_t* q_codes;
  const uint32_t* k_codes;
  int32_t* idx;
  int32_t* dist;
  int Hq, Hkv, g;
  int64_t cap, lo, C;
  int k_eff, top_k;
  int p0, P;
  int64_t per_block;
  int nbins, max_seg;
  uint32_t* sync;  // [pairs][2]: arrivals, departures
  uint32_t* hist;  // [pairs][nbins]
  uint32_t* cum;   // [pairs][max_seg][nbins]
  int32_t* status;
  uint64_t wait_ns;
  int skip_arrive;
};

template <int W, int NP>
struct Planes {
  uint32_t C[NP][W];
  uint32_t U[NP][W];
};

// Bit-sliced counters: C planes count the query codes' ones, U planes their zeros.
template <int W, int NP>
__device__ __forceinline__ void build_planes(const uint32_t* __restrict__ qc, int g, Planes<W, NP>& p) {
#pragma unroll
  for (int b = 0; b < NP; ++b)
#pragma unroll
    for (int w = 0; w < W; ++w) p.C[b][w] = p.U[b][w] = 0u;
  for (int h = 0; h < g; ++h) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const uint32_t q = __ldg(qc + h * W + w);
      uint32_t carry = q;
#pragma unroll
      for (int b = 0; b < NP; ++b) {
        const uint32_t t = p.C[b][w] & carry;
        p.C[b][w] ^= carry;
        carry = t;
      }
      carry = ~q;
#pragma unroll
      for (int b = 0; b < NP; ++b) {
        const uint32_t t = p.U[b][w] & carry;
        p.U[b][w] ^= carry;
        carry = t;
      }
    }
  }
}

// s = a + b on bit-sliced numbers of NB planes (ripple of full adders).
template <int NB>
__device__ __forceinline__ void add_planes(const uint32_t (&a)[NB], const uint32_t (&b)[NB], uint32_t (&s)[NB + 1]) {
  uint32_t c = 0u;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const uint32_t x = a[i], y = b[i];
    s[i] = x ^ y ^ c;
    c = (x & y) | (c & (x ^ y));
  }
  s[NB] = c;
}

template <int L>
__device__ __forceinline__ int weighted_popc(const uint32_t (&s)[L]) {
  int r = 0;
#pragma unroll
  for (int b = 0; b < L; ++b) r += __popc(s[b]) << b;
  return r;
}

template <int W, int NP>
__device__ __forceinline__ int token_distance(const uint32_t (&ck)[W], const Planes<W, NP>& p) {
  uint32_t v[W][NP];
#pragma unroll
  for (int w = 0; w < W; ++w)
#pragma unroll
    for (int b = 0; b < NP; ++b) v[w][b] = (ck[w] & p.U[b][w]) | (~ck[w] & p.C[b][w]);
  if constexpr (W == 2) {
    uint32_t s[NP + 1];
    add_planes<NP>(v[0], v[1], s);
    return weighted_popc<NP + 1>(s);
  } else {
    static_assert(W == 4, "codes of 64 or 128 bits");
    uint32_t s01[NP + 1], s23[NP + 1], s[NP + 2];
    add_planes<NP>(v[0], v[1], s01);
    add_planes<NP>(v[2], v[3], s23);
    add_planes<NP + 1>(s01, s23, s);
    return weighted_popc<NP + 2>(s);
  }
}

// In-place inclusive prefix sum over a[0, n) in shared memory.
__device__ void block_inclusive_scan(uint32_t* a, int n, uint32_t* warp_tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kThreads - 1) / kThreads;
  const int beg = min(tid * per, n), end = min(beg + per, n);
  uint32_t s = 0;
  for (int i = beg; i < end; ++i) s += a[i];
  uint32_t x = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  uint32_t run = x - s;
  for (int w = 0; w < warp; ++w) run += warp_tmp[w];
  for (int i = beg; i < end; ++i) {
    run += a[i];
    a[i] = run;
  }
  __syncthreads();
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* warp_tmp) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) warp_tmp[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t s = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += warp_tmp[w];
  return s;
}

template <int W, int NP>
__global__ void __launch_bounds__(kThreads, kMaxBlocksPerSM) scan_select_kernel(RetrieveArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem_raw);
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(hist_s + ((a.nbins + 3) & ~3));
  __shared__ uint32_t warp_tmp[kWarps];
  __shared__ uint32_t warp_lt[kWarps], warp_eq[kWarps];
  __shared__ int s_flag, s_T;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t C = a.C;
  const int64_t U = (int64_t)a.P * C;
  const int64_t f0 = (int64_t)blockIdx.x * a.per_block;
  const int64_t f1 = min(f0 + a.per_block, U);
  if (f0 >= f1) return;
  const int pa = (int)(f0 / C), pb = (int)((f1 - 1) / C);

  // ---------------- phase A: distances, histograms ----------------
  int64_t soff = 0;
  for (int pl = pa; pl <= pb; ++pl) {
    const int p = a.p0 + pl;
    const int64_t s0 = max(f0, pl * C) - pl * C, s1 = min(f1, (pl + 1) * C) - pl * C;
    const int seg = (int)(blockIdx.x - (pl * C) / a.per_block);
    for (int i = tid; i < a.nbins; i += kThreads) hist_s[i] = 0u;
    const int b = p / a.Hkv, kvh = p % a.Hkv;
    Planes<W, NP> planes;
    build_planes<W, NP>(a.q_codes + ((int64_t)b * a.Hq + (int64_t)kvh * a.g) * W, a.g, planes);
    __syncthreads();
    const uint32_t* kc = a.k_codes + ((int64_t)p * a.cap + a.lo) * W;
    uint16_t* dseg = dist_s + soff;
    for (int64_t base = s0; base < s1; base += kThreads * kUnroll) {
      uint32_t ck[kUnroll][W];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads + tid;
        if (i < s1) ld_stream(kc + i * W, ck[u]);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads + tid;
        if (i < s1) {
          const int Dv = token_distance<W, NP>(ck[u], planes);
          dseg[i - s0] = (uint16_t)Dv;
          atomicAdd(&hist_s[Dv], 1u);
        }
      }
    }
    __syncthreads();
    block_inclusive_scan(hist_s, a.nbins, warp_tmp);
    uint32_t* cum_out = a.cum + ((int64_t)p * a.max_seg + seg) * a.nbins;
    uint32_t* hist_out = a.hist + (int64_t)p * a.nbins;
    for (int v = tid; v < a.nbins; v += kThreads) {
      const uint32_t c = hist_s[v];
      const uint32_t n = c - (v > 0 ? hist_s[v - 1] : 0u);
      cum_out[v] = c;
      if (n) atomicAdd(&hist_out[v], n);
    }
    soff += s1 - s0;
    __syncthreads();
  }
  if (tid == 0) {
    __threadfence();
    if (!(a.skip_arrive && blockIdx.x == 0))
      for (int pl = pa; pl <= pb; ++pl) atomicAdd(&a.sync[2 * (a.p0 + pl)], 1u);
  }

  // ---------------- phase B: threshold, ordered compaction ----------------
  soff = 0;
  for (int pl = pa; pl <= pb; ++pl) {
    const int p = a.p0 + pl;
    const int64_t s0 = max(f0, pl * C) - pl * C, s1 = min(f1, (pl + 1) * C) - pl * C;
    const int first = (int)((pl * C) / a.per_block);
    const int last = (int)(((pl + 1) * C - 1) / a.per_block);
    const int nseg = last - first + 1, seg = (int)blockIdx.x - first;
    if (tid == 0) {
      const uint64_t t0 = globaltimer_ns();
      int ok = 1;
      for (uint32_t it = 0; ld_acquire_gpu(&a.sync[2 * p]) < (uint32_t)nseg; ++it) {
        if (globaltimer_ns() - t0 > a.wait_ns || it > (1u << 28)) {
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
      __threadfence();
      s_flag = ok;
    }
    __syncthreads();
    if (s_flag) {
      const uint32_t* hist_in = a.hist + (int64_t)p * a.nbins;
      for (int v = tid; v < a.nbins; v += kThreads) hist_s[v] = __ldcg(hist_in + v);
      if (tid == 0) s_T = a.nbins - 1;
      __syncthreads();
      block_inclusive_scan(hist_s, a.nbins, warp_tmp);
      const uint32_t k_eff = (uint32_t)a.k_eff;
      for (int v = tid; v < a.nbins; v += kThreads)
        if (hist_s[v] >= k_eff && (v == 0 || hist_s[v - 1] < k_eff)) s_T = v;
      __syncthreads();
      const int T = s_T;
      const uint32_t below = T > 0 ? hist_s[T - 1] : 0u;
      const uint32_t ties_needed = k_eff - below;
      // selected-before counts from the lower segments of this pair
      uint32_t lt = 0, le = 0;
      for (int s = tid; s < seg; s += kThreads) {
        const uint32_t* cs = a.cum + ((int64_t)p * a.max_seg + s) * a.nbins;
        lt += T > 0 ? __ldcg(cs + T - 1) : 0u;
        le += __ldcg(cs + T);
      }
      const uint32_t lower_lt = block_sum(lt, warp_tmp);
      const uint32_t lower_eq = block_sum(le, warp_tmp) - lower_lt;
      const uint32_t quota = ties_needed > lower_eq ? ties_needed - lower_eq : 0u;
      const uint32_t sel_base = lower_lt + min(lower_eq, ties_needed);
      // ordered compaction of this segment
      const int64_t len = s1 - s0;
      const int64_t per_w = ((len + kWarps * 32 - 1) / (kWarps * 32)) * 32;
      const int64_t w0 = min((int64_t)warp * per_w, len), w1 = min(w0 + per_w, len);
      const uint16_t* dseg = dist_s + soff;
      uint32_t clt = 0, ceq = 0;
      for (int64_t c = w0; c < w1; c += 32) {
        const int64_t i = c + lane;
        const int Dv = i < w1 ? (int)dseg[i] : 0x7fffffff;
        clt += __popc(__ballot_sync(0xffffffffu, Dv < T));
        ceq += __popc(__ballot_sync(0xffffffffu, Dv == T));
      }
      if (lane == 0) {
        warp_lt[warp] = clt;
        warp_eq[warp] = ceq;
      }
      __syncthreads();
      uint32_t ex_lt = 0, ex_eq = 0;
      for (int w = 0; w < warp; ++w) {
        ex_lt += warp_lt[w];
        ex_eq += warp_eq[w];
      }
      uint32_t run_eq = ex_eq, run_sel = ex_lt + min(ex_eq, quota);
      int32_t* idx_out = a.idx + (int64_t)p * a.top_k + sel_base;
      int32_t* dist_out = a.dist ? a.dist + (int64_t)p * a.top_k + sel_base : nullptr;
      const uint32_t below_lane = lanemask_lt();
      for (int64_t c = w0; c < w1; c += 32) {
        const int64_t i = c + lane;
        const int Dv = i < w1 ? (int)dseg[i] : 0x7fffffff;
        const uint32_t meq = __ballot_sync(0xffffffffu, Dv == T);
        const bool take_eq = Dv == T && run_eq + __popc(meq & below_lane) < quota;
        const bool sel = Dv < T || take_eq;
        const uint32_t msel = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const uint32_t pos = run_sel + __popc(msel & below_lane);
          if (sel_base + pos < k_eff) {
            idx_out[pos] = (int32_t)(a.lo + s0 + i);
            if (dist_out) dist_out[pos] = Dv;
          } else {
            report(a.status, HKV_ERR_DEVICE_RANGE);  // unreachable when the counts agree
          }
        }
        run_eq += __popc(meq);
        run_sel += __popc(msel);
      }
    } else if (tid == 0) {
      report(a.status, HKV_ERR_TIMEOUT);
    }
    soff += s1 - s0;
    // depart; the last block out of this pair cleans its scratch
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      s_flag = atomicAdd(&a.sync[2 * p + 1], 1u) == (uint32_t)(nseg - 1);
    }
    __syncthreads();
    if (s_flag) {
      __threadfence();
      uint32_t* hist_out = a.hist + (int64_t)p * a.nbins;
      for (int v = tid; v < a.nbins; v += kThreads) hist_out[v] = 0u;
      for (int i = a.k_eff + tid; i < a.top_k; i += kThreads) {
        a.idx[(int64_t)p * a.top_k + i] = -1;
        if (a.dist) a.dist[(int64_t)p * a.top_k + i] = -1;
      }
      if (tid == 0) {
        a.sync[2 * p] = 0u;
        a.sync[2 * p + 1] = 0u;
      }
    }
    __syncthreads();
  }
}

using KernelFn = void (*)(RetrieveArgs);

KernelFn pick_kernel(int words, int np) {
#define HKV_PICK(W, NPV) \
  if (words == W && np == NPV) return scan_select_kernel<W, NPV>;
  HKV_PICK(2, 1) HKV_PICK(2, 2) HKV_PICK(2, 3) HKV_PICK(2, 4) HKV_PICK(2, 5)
  HKV_PICK(4, 1) HKV_PICK(4, 2) HKV_PICK(4, 3) HKV_PICK(4, 4) HKV_PICK(4, 5)
#undef HKV_PICK
  return nullptr;
}

int bit_length(int v) {
  int n = 0;
  while (v) {
    ++n;
    v >>= 1;
  }
  return n;
}

struct Plan {
  int nbins, np;
  int64_t C, lo;
  int k_eff;
  int pairs_per_launch;
  int64_t per_block;  // for a full batch of pairs_per_launch pairs
  int max_seg;
  int blocks_per_sm;
  size_t smem;
  size_t ws_sync, ws_hist, ws_cum, ws_total;
};

int make_plan(const RetrieveShape& s, Plan& pl) {
  const int g = s.Hq / s.Hkv;
  const int bits = s.words * 32;
  const Window w = window(s.N, s.n_sink, s.n_local);
  pl.C = w.C;
  pl.lo = w.sink_end;
  pl.k_eff = (int)(s.top_k < w.C ? s.top_k : w.C);
  pl.nbins = g * bits + 1;
  pl.np = bit_length(g);
  pl.smem = align_up(sizeof(uint32_t) * ((pl.nbins + 3) & ~3), 16) + sizeof(uint16_t) * kMaxTokensPerBlock;
  KernelFn k = pick_kernel(s.words, pl.np);
  if (k == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no scan kernel for %d-bit codes and group size %d", bits, g);
  int per_sm = 0;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, pl.smem);
  if (e != cudaSuccess) return cuda_check(e, "scan occupancy");
  if (per_sm > kMaxBlocksPerSM) per_sm = kMaxBlocksPerSM;
  if (per_sm < 1) return fail(HKV_ERR_UNSUPPORTED, "scan kernel does not fit on an SM");
  pl.blocks_per_sm = per_sm;
  const int64_t gmax = (int64_t)sm_count() * per_sm;
  const int P = s.B * s.Hkv;
  const int64_t C = pl.C > 0 ? pl.C : 1;
  if (C > gmax * kMaxTokensPerBlock)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates exceed one launch (%lld)", (long long)C,
                (long long)(gmax * kMaxTokensPerBlock));
  int64_t ppl = P;
  if ((int64_t)P * C > gmax * kMaxTokensPerBlock) ppl = (gmax * kMaxTokensPerBlock) / C;
  if (ppl < 1) ppl = 1;
  pl.pairs_per_launch = (int)ppl;
  const int64_t Uf = ppl * C;
  int64_t per = ceil_div(Uf, gmax);
  if (per < kMinTokensPerBlock) per = kMinTokensPerBlock;
  per = ceil_div(per, 32) * 32;
  if (per > kMaxTokensPerBlock) per = kMaxTokensPerBlock;
  pl.per_block = per;
  // Smaller (last) batches use the same per_block, so this bounds them too.
  pl.max_seg = (int)(ceil_div(C, per) + 1);
  pl.ws_sync = align_up(sizeof(uint32_t) * 2 * P, 256);
  pl.ws_hist = align_up(sizeof(uint32_t) * (size_t)P * pl.nbins, 256);
  pl.ws_cum = align_up(sizeof(uint32_t) * (size_t)P * pl.max_seg * pl.nbins, 256);
  pl.ws_total = pl.ws_sync + pl.ws_hist + pl.ws_cum;
  return HKV_OK;
}

}  // namespace

size_t retrieve_ws_bytes(const RetrieveShape& s) {
  Plan pl;
  if (make_plan(s, pl) != HKV_OK) return 0;
  return pl.ws_total;
}

int launch_retrieve(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                    int32_t* idx, int32_t* dist, void* ws, size_t ws_bytes, int32_t* status,
                    cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  Plan pl;
  int rc = make_plan(s, pl);
  if (rc != HKV_OK) return rc;
  if (pl.k_eff == 0) {
    rc = cuda_check(cudaMemsetAsync(idx, 0xff, sizeof(int32_t) * (size_t)P * s.top_k, st), "idx fill");
    if (rc == HKV_OK && dist)
      rc = cuda_check(cudaMemsetAsync(dist, 0xff, sizeof(int32_t) * (size_t)P * s.top_k, st), "dist fill");
    return rc;
  }
  if (ws_bytes < pl.ws_total || ws == nullptr)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, pl.ws_total);
  unsigned char* base = static_cast<unsigned char*>(ws);
  RetrieveArgs a;
  a.q_codes = q_codes;
  a.k_codes = k_codes;
  a.idx = idx;
  a.dist = dist;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = s.Hq / s.Hkv;
  a.cap = s.cap;
  a.lo = pl.lo;
  a.C = pl.C;
  a.k_eff = pl.k_eff;
  a.top_k = s.top_k;
  a.per_block = pl.per_block;
  a.nbins = pl.nbins;
  a.max_seg = pl.max_seg;
  a.sync = reinterpret_cast<uint32_t*>(base);
  a.hist = reinterpret_cast<uint32_t*>(base + pl.ws_sync);
  a.cum = reinterpret_cast<uint32_t*>(base + pl.ws_sync + pl.ws_hist);
  a.status = status;
  a.wait_ns = wait_limit_ns();
  a.skip_arrive = (debug_flags() & kDebugSkipArrive) ? 1 : 0;
  KernelFn k = pick_kernel(s.words, pl.np);
  for (int p0 = 0; p0 < P; p0 += pl.pairs_per_launch) {
    a.p0 = p0;
    a.P = P - p0 < pl.pairs_per_launch ? P - p0 : pl.pairs_per_launch;
    const int64_t grid = ceil_div((int64_t)a.P * pl.C, pl.per_block);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = grid > 1 ? 1 : 0;
    rc = cuda_check(cudaLaunchKernelEx(&cfg, k, a), "scan/select launch");
    if (rc != HKV_OK) return rc;
  }
  return HKV_OK;
}

}  // namespace hkv
