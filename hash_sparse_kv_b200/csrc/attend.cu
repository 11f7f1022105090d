// Sparse decode attention over sink + selected + local rows, and the
// log-sum-exp merge of partial results (S6, S7, S8).
//
// Spotlight Attention ("Approach"): exact attention over only the retrieved
// tokens, with sink and local-window tokens kept.  RetrievalAttention
// ("Summary", "Approach"): a fixed resident pattern and the retrieved part are
// attended separately and their partial results combined by exact
// log-sum-exp rescaling.
//
// The rows of KV head j form a virtual list [sink | idx slots | local].  Each
// block takes a contiguous slice of that list (a split), gathers the K and V
// rows once for all g query heads of the group, and produces a partial result
// (m_h, l_h, acc_h) with m_h the max logit, l_h = sum exp(z - m_h) and
// acc_h = sum exp(z - m_h) V.  The last block of a KV head to finish (ticket
// counter in the workspace) merges the splits:
//   M = max_s m_s,  L = sum_s l_s e^{m_s - M},  out = sum_s acc_s e^{m_s - M} / L,
//   lse = M + log L.
// Probabilities and accumulators stay fp32.  This SIMT kernel serves fp32
// caches; bf16 caches go to the tensor-core kernel (launch_sattend).
#include <math.h>

#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRows = 64;   // rows per split
constexpr int kMaxGroup = 16;  // query heads per KV head
constexpr int kKP = kHeadDim + 1;
constexpr int kPartStride = kHeadDim + 2;  // m, l, acc[128]

struct AttendArgs {
  const void* q;
  const void* K;
  const void* V;
  const int32_t* idx;
  float* out;
  float* lse;
  float* part;       // [pairs][splits][g][kPartStride]
  uint32_t* ticket;  // [pairs]
  int Hq, Hkv, g;
  int64_t cap, N;
  int top_k;
  int64_t sink_n, local_start, local_n;
  float scale;
  int rows_per_split, splits;
  int32_t* status;
  PageMap pm;  // paged K/V pools when PAGED
};

// K and V rows of token t of pair (b, kvh): contiguous [B, Hkv, cap, 128], or
// slot t % page_size of pool page table[b, t / page_size] ([num_pages, Hkv,
// page_size, 128]); -1 when that page id is outside the pool.
template <bool PAGED>
__device__ __forceinline__ int64_t kv_row_of(const AttendArgs& a, int b, int kvh, int p, int64_t t) {
  if constexpr (PAGED) {
    const int pg = a.pm.table[(int64_t)b * a.pm.max_pages + t / a.pm.page_size];
    if (pg < 0 || pg >= a.pm.num_pages) return -1;
    return ((int64_t)pg * a.Hkv + kvh) * a.pm.page_size + t % a.pm.page_size;
  } else {
    return (int64_t)p * a.cap + t;
  }
}

template <typename T, bool PAGED>
__global__ void __launch_bounds__(kThreads) attend_kernel(AttendArgs a) {
  extern __shared__ __align__(16) float smem[];
  float* q_s = smem;                          // [g][128]
  float* K_s = q_s + kMaxGroup * kHeadDim;    // [rows][129]
  float* V_s = K_s + kMaxRows * kKP;          // [rows][128]
  float* z_s = V_s + kMaxRows * kHeadDim;     // [g][rows]
  __shared__ int tok_s[kMaxRows];
  __shared__ float m_s[kMaxGroup], l_s[kMaxGroup];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = blockIdx.x / a.splits, sp = blockIdx.x % a.splits;
  const int b = p / a.Hkv, kvh = p % a.Hkv, g = a.g;
  const int64_t Rv = a.sink_n + a.top_k + a.local_n;
  const int64_t v0 = (int64_t)sp * a.rows_per_split;
  const int nrows = (int)max((int64_t)0, min((int64_t)a.rows_per_split, Rv - v0));

  const T* qp = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)kvh * g) * kHeadDim;
  const T* Kb = static_cast<const T*>(a.K);
  const T* Vb = static_cast<const T*>(a.V);

  for (int i = tid; i < nrows; i += kThreads) {
    const int64_t v = v0 + i;
    int64_t t;
    if (v < a.sink_n) {
      t = v;
    } else if (v < a.sink_n + a.top_k) {
      t = a.idx[(int64_t)p * a.top_k + (v - a.sink_n)];
      if (t >= a.N) {
        report(a.status, HKV_ERR_DEVICE_RANGE);
        t = -1;
      }
    } else {
      t = a.local_start + (v - a.sink_n - a.top_k);
    }
    if (PAGED && t >= 0 && kv_row_of<PAGED>(a, b, kvh, p, t) < 0) {
      report(a.status, HKV_ERR_DEVICE_RANGE);
      t = -1;
    }
    tok_s[i] = t < 0 ? -1 : (int)t;
  }
  for (int i = tid; i < g * (kHeadDim / 4); i += kThreads) {
    const int h = i / (kHeadDim / 4), c = (i % (kHeadDim / 4)) * 4;
    const float4 v = load4_f32(qp + (int64_t)h * kHeadDim + c);
    *reinterpret_cast<float4*>(&q_s[h * kHeadDim + c]) = v;
  }
  __syncthreads();
  {
    // every K/V load of this thread is in flight before the first shared store
    constexpr int EPC = 16 / sizeof(T), CPR = kHeadDim / EPC, kPer = kMaxRows * CPR / kThreads;
    uint4 kr[kPer], vr[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kThreads, r = i / CPR, c = i % CPR;
      const int t = r < nrows ? tok_s[r] : -1;
      kr[u] = vr[u] = make_uint4(0u, 0u, 0u, 0u);
      if (t >= 0) {
        const int64_t row = kv_row_of<PAGED>(a, b, kvh, p, t);
        kr[u] = __ldg(reinterpret_cast<const uint4*>(Kb + row * kHeadDim) + c);
        vr[u] = __ldg(reinterpret_cast<const uint4*>(Vb + row * kHeadDim) + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kThreads, r = i / CPR, c = i % CPR;
      if (r >= nrows) continue;
      const T* ke = reinterpret_cast<const T*>(&kr[u]);
      const T* ve = reinterpret_cast<const T*>(&vr[u]);
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        K_s[r * kKP + c * EPC + e] = to_f32(ke[e]);
        V_s[r * kHeadDim + c * EPC + e] = to_f32(ve[e]);
      }
    }
  }
  __syncthreads();
  // logits z[h][r] = scale * q_h . K_r  (-inf for empty slots)
  for (int o = tid; o < g * nrows; o += kThreads) {
    const int h = o / nrows, r = o % nrows;
    float z = -INFINITY;
    if (tok_s[r] >= 0) {
      const float* qh = q_s + h * kHeadDim;
      const float* kr = K_s + r * kKP;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
      for (int c = 0; c < kHeadDim; c += 4) {
        a0 = fmaf(qh[c], kr[c], a0);
        a1 = fmaf(qh[c + 1], kr[c + 1], a1);
        a2 = fmaf(qh[c + 2], kr[c + 2], a2);
        a3 = fmaf(qh[c + 3], kr[c + 3], a3);
      }
      z = ((a0 + a1) + (a2 + a3)) * a.scale;
    }
    z_s[h * kMaxRows + r] = z;
  }
  __syncthreads();
  // per-head max and sum; z_s becomes the unnormalised probabilities
  for (int h = warp; h < g; h += kThreads / 32) {
    float m = -INFINITY;
    for (int r = lane; r < nrows; r += 32) m = fmaxf(m, z_s[h * kMaxRows + r]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int r = lane; r < nrows; r += 32) {
      const float z = z_s[h * kMaxRows + r];
      const float e = z == -INFINITY ? 0.f : expf(z - m);
      z_s[h * kMaxRows + r] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      m_s[h] = m;
      l_s[h] = l;
    }
  }
  __syncthreads();
  float* part = a.part + ((int64_t)p * a.splits + sp) * g * kPartStride;
  for (int o = tid; o < g * kHeadDim; o += kThreads) {
    const int h = o / kHeadDim, c = o % kHeadDim;
    const float* zh = z_s + h * kMaxRows;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int r = 0;
    for (; r + 4 <= nrows; r += 4) {
      a0 = fmaf(zh[r], V_s[r * kHeadDim + c], a0);
      a1 = fmaf(zh[r + 1], V_s[(r + 1) * kHeadDim + c], a1);
      a2 = fmaf(zh[r + 2], V_s[(r + 2) * kHeadDim + c], a2);
      a3 = fmaf(zh[r + 3], V_s[(r + 3) * kHeadDim + c], a3);
    }
    for (; r < nrows; ++r) a0 = fmaf(zh[r], V_s[r * kHeadDim + c], a0);
    const float acc = (a0 + a1) + (a2 + a3);
    part[h * kPartStride + 2 + c] = acc;
    if (c == 0) {
      part[h * kPartStride + 0] = m_s[h];
      part[h * kPartStride + 1] = l_s[h];
    }
  }
  // the last split of this KV head merges all splits
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&a.ticket[p], 1u) == (uint32_t)(a.splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* parts = a.part + (int64_t)p * a.splits * g * kPartStride;
  float* w_s = K_s;  // [splits][g] merge weights, reusing the K tile
  for (int h = warp; h < g; h += kThreads / 32) {
    float M = -INFINITY;
    for (int s = lane; s < a.splits; s += 32) M = fmaxf(M, __ldcg(parts + ((int64_t)s * g + h) * kPartStride));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    for (int s = lane; s < a.splits; s += 32) {
      const float* ps = parts + ((int64_t)s * g + h) * kPartStride;
      const float ms = __ldcg(ps);
      const float w = (ms == -INFINITY) ? 0.f : expf(ms - M);
      w_s[s * g + h] = w;
      L = fmaf(__ldcg(ps + 1), w, L);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) {
      m_s[h] = M;
      l_s[h] = L;
    }
  }
  __syncthreads();
  for (int o = tid; o < g * (kHeadDim / 4); o += kThreads) {
    const int h = o / (kHeadDim / 4), c = (o % (kHeadDim / 4)) * 4;
    const float L = l_s[h];
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    if (L > 0.f) {
#pragma unroll 4
      for (int s = 0; s < a.splits; ++s) {
        const float w = w_s[s * g + h];
        const float* ps = parts + ((int64_t)s * g + h) * kPartStride + 2 + c;
        const float2 x0 = __ldcg(reinterpret_cast<const float2*>(ps));
        const float2 x1 = __ldcg(reinterpret_cast<const float2*>(ps + 2));
        O.x = fmaf(x0.x, w, O.x);
        O.y = fmaf(x0.y, w, O.y);
        O.z = fmaf(x1.x, w, O.z);
        O.w = fmaf(x1.y, w, O.w);
      }
      const float inv = 1.f / L;
      O.x *= inv;
      O.y *= inv;
      O.z *= inv;
      O.w *= inv;
    }
    const int64_t orow = (int64_t)b * a.Hq + (int64_t)kvh * g + h;
    *reinterpret_cast<float4*>(a.out + orow * kHeadDim + c) = O;
    if (c == 0 && a.lse != nullptr) a.lse[orow] = L > 0.f ? m_s[h] + logf(L) : -INFINITY;
  }
  if (tid == 0) a.ticket[p] = 0u;
}

__global__ void lse_merge_kernel(int rows, int d, const float* __restrict__ o1, const float* __restrict__ lse1,
                                 const float* __restrict__ o2, const float* __restrict__ lse2,
                                 float* __restrict__ out, float* __restrict__ lse_out) {
  const int64_t total = (int64_t)rows * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / d;
    const float a = lse1[r], b = lse2[r];
    const float m = fmaxf(a, b);
    float o = 0.f, l = -INFINITY;
    if (m != -INFINITY) {
      const float w1 = a == -INFINITY ? 0.f : expf(a - m);
      const float w2 = b == -INFINITY ? 0.f : expf(b - m);
      const float s = w1 + w2;
      o = (w1 * o1[i] + w2 * o2[i]) / s;
      l = m + logf(s);
    }
    out[i] = o;
    if (lse_out != nullptr && i % d == 0) lse_out[r] = l;
  }
}

struct AttendPlan {
  int64_t Rv;
  int rows_per_split, splits;
  size_t smem, ws_part, ws_ticket, ws_total;
};

AttendPlan make_plan(const AttendShape& s) {
  AttendPlan pl;
  const Window w = window(s.N, s.n_sink, s.n_local);
  const int g = s.Hq / s.Hkv;
  const int P = s.B * s.Hkv;
  pl.Rv = w.sink_end + s.top_k + (s.N - w.local_start);
  // Aim for about one block per SM, 32..kMaxRows rows per block (the merge
  // reads every split, so fewer, fuller splits keep it short).
  const int64_t target = (int64_t)sm_count();
  int64_t splits = ceil_div(target, P > 0 ? P : 1);
  int64_t rps = ceil_div(pl.Rv > 0 ? pl.Rv : 1, splits);
  if (rps > kMaxRows) rps = kMaxRows;
  if (rps < 32) rps = 32;
  pl.rows_per_split = (int)rps;
  pl.splits = (int)ceil_div(pl.Rv > 0 ? pl.Rv : 1, rps);
  pl.smem = sizeof(float) * (kMaxGroup * kHeadDim + kMaxRows * kKP + kMaxRows * kHeadDim + kMaxGroup * kMaxRows);
  pl.ws_part = align_up(sizeof(float) * (size_t)P * pl.splits * g * kPartStride, 256);
  pl.ws_ticket = align_up(sizeof(uint32_t) * (size_t)P, 256);
  pl.ws_total = pl.ws_part + pl.ws_ticket;
  return pl;
}

}  // namespace

// A workspace sized here serves both element types (the bf16 plan is the
// tensor-core kernel's).
size_t attend_ws_bytes(const AttendShape& s) {
  const size_t simt = make_plan(s).ws_total, tc = sattend_ws_bytes(s);
  return simt > tc ? simt : tc;
}

int launch_attend(const AttendShape& s, const void* q, const void* K, const void* V,
                  const int32_t* idx, float scale, float* out, float* lse, void* ws,
                  size_t ws_bytes, int32_t* status, cudaStream_t st, const PageMap* pm) {
  const int P = s.B * s.Hkv;
  if (P == 0) return HKV_OK;
  if (s.dtype == HKV_BF16) return launch_sattend(s, q, K, V, idx, scale, out, lse, ws, ws_bytes, status, st, pm);
  const AttendPlan pl = make_plan(s);
  if ((int64_t)pl.splits * (s.Hq / s.Hkv) > (int64_t)kMaxRows * kKP)
    return fail(HKV_ERR_UNSUPPORTED, "%lld attended rows per KV head is too many", (long long)pl.Rv);
  if (ws == nullptr || ws_bytes < pl.ws_total)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, pl.ws_total);
  const Window w = window(s.N, s.n_sink, s.n_local);
  AttendArgs a;
  a.q = q;
  a.K = K;
  a.V = V;
  a.idx = idx;
  a.out = out;
  a.lse = lse;
  a.part = reinterpret_cast<float*>(ws);
  a.ticket = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + pl.ws_part);
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = s.Hq / s.Hkv;
  a.cap = s.cap;
  a.N = s.N;
  a.top_k = s.top_k;
  a.sink_n = w.sink_end;
  a.local_start = w.local_start;
  a.local_n = s.N - w.local_start;
  a.scale = scale;
  a.rows_per_split = pl.rows_per_split;
  a.splits = pl.splits;
  a.status = status;
  a.pm = pm != nullptr ? *pm : PageMap{};
  const int grid = P * pl.splits;
  using Fn = void (*)(AttendArgs);
  Fn k = s.dtype == HKV_BF16 ? (pm != nullptr ? attend_kernel<__nv_bfloat16, true> : attend_kernel<__nv_bfloat16, false>)
                             : (pm != nullptr ? attend_kernel<float, true> : attend_kernel<float, false>);
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
  k<<<grid, kThreads, pl.smem, st>>>(a);
  return cuda_check(cudaGetLastError(), "attend launch");
}

int launch_lse_merge(int rows, int d, const float* o1, const float* lse1, const float* o2,
                     const float* lse2, float* out, float* lse_out, cudaStream_t st) {
  const int64_t total = (int64_t)rows * d;
  if (total == 0) return HKV_OK;
  int64_t grid = ceil_div(total, 256);
  if (grid > 8L * sm_count()) grid = 8L * sm_count();
  lse_merge_kernel<<<(int)grid, 256, 0, st>>>(rows, d, o1, lse1, o2, lse2, out, lse_out);
  return cuda_check(cudaGetLastError(), "lse merge launch");
}

}  // namespace hkv
