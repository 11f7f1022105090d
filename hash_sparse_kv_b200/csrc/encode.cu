// Hash encoders: vectors -> packed sign codes.
//
//   LSH  (HashEvict, "Abstract"): bit j = [ (R x)_j > 0 ], R Gaussian [bits, d]
//   MLP  (Spotlight Attention, "Approach"): bit j = [ (W2 SiLU(W1 x + b1) + b2)_j > 0 ]
//   SIGN (Self-Indexing KVCache, "Abstract"): bit i = [ x_i > 0 ], plus ||x||_2 as fp16
//
// Bits are packed least-significant first: bit j -> word j / 32, position j % 32.
// In the projection kernels lane l of a warp owns bits {l + 32 i}, so word i of
// a row is exactly the warp ballot of (y_{l + 32 i} > 0).
#include <cooperative_groups.h>
#include <cstdio>

#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 256;
constexpr int64_t kFewRows = 2048;  // up to this many rows use the per-16-row projection kernel

// ---------------------------------------------------------------- LSH -----
// Tile of 64 rows per pass; warp w owns rows [8w, 8w + 8); lane l owns bits
// {l + 32 i : i < BITS / 32}.  R^T and the x tile (transposed) sit in shared
// memory as fp32; products and sums are fp32.
template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads, 2)
lsh_encode_kernel(const T* __restrict__ x, const T* __restrict__ R, RowMap m,
                  uint32_t* __restrict__ codes) {
  constexpr int D = kHeadDim, ROWS = 64, TB = BITS / 32, XP = ROWS + 4;
  extern __shared__ __align__(16) float smem[];
  float* RT = smem;          // [D][BITS]
  float* xT = RT + D * BITS;  // [D][XP]
  for (int i = threadIdx.x; i < BITS * D; i += kThreads) {
    const int j = i % BITS, k = i / BITS;
    RT[k * BITS + j] = to_f32(R[(int64_t)j * D + k]);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (m.rows + ROWS - 1) / ROWS;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t r0 = tile * ROWS;
    __syncthreads();
    for (int i = threadIdx.x; i < ROWS * (D / 4); i += kThreads) {
      const int r = i / (D / 4), k4 = (i % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + r < m.rows) v = load4_f32(x + m.x_off(r0 + r) + k4);
      xT[(k4 + 0) * XP + r] = v.x;
      xT[(k4 + 1) * XP + r] = v.y;
      xT[(k4 + 2) * XP + r] = v.z;
      xT[(k4 + 3) * XP + r] = v.w;
    }
    __syncthreads();
    float acc[8][TB];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int i = 0; i < TB; ++i) acc[r][i] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float4 xa = *reinterpret_cast<const float4*>(&xT[k * XP + warp * 8]);
      const float4 xb = *reinterpret_cast<const float4*>(&xT[k * XP + warp * 8 + 4]);
      const float xr[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        const float rv = RT[k * BITS + lane + 32 * i];
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r][i] = fmaf(xr[r], rv, acc[r][i]);
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int64_t row = r0 + warp * 8 + r;
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        const uint32_t word = __ballot_sync(0xffffffffu, acc[r][i] > 0.f);
        if (lane == i && row < m.rows) codes[m.c_off(row) + i] = word;
      }
    }
  }
}

// Few rows (query heads of a decode step, short appends): 16 rows per block,
// R staged once per block with padded rows (odd word stride, so the lanes of
// a warp -- consecutive bits j -- read distinct banks).  Thread t owns bit
// j = t % BITS of rows {t / BITS + SLOTS * i}.
template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads)
lsh_rows_kernel(const T* __restrict__ x, const T* __restrict__ R, RowMap m, uint32_t* __restrict__ codes) {
  constexpr int D = kHeadDim, ROWS = 16, SLOTS = kThreads / BITS, RPT = ROWS / SLOTS;
  constexpr int RP = D + (sizeof(T) == 2 ? 2 : 1);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* x_s = reinterpret_cast<float*>(smem_raw);            // [ROWS][D]
  T* R_s = reinterpret_cast<T*>(x_s + ROWS * D);               // [BITS][RP]
  constexpr int V = 16 / sizeof(T);
  for (int i = threadIdx.x; i < BITS * (D / V); i += kThreads) {
    const int j = i / (D / V), c = (i % (D / V)) * V;
    const uint4 raw = *reinterpret_cast<const uint4*>(R + (int64_t)j * D + c);
    const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int u = 0; u < V; ++u) R_s[j * RP + c + u] = e[u];
  }
  const int64_t r0 = (int64_t)blockIdx.x * ROWS;
  for (int i = threadIdx.x; i < ROWS * (D / 4); i += kThreads) {
    const int r = i / (D / 4), c = (i % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < m.rows) v = load4_f32(x + m.x_off(r0 + r) + c);
    *reinterpret_cast<float4*>(&x_s[r * D + c]) = v;
  }
  __syncthreads();
  const int j = threadIdx.x % BITS, slot = threadIdx.x / BITS, lane = threadIdx.x & 31;
  float acc[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; k += 2) {
    const float r_a = to_f32(R_s[j * RP + k]), r_b = to_f32(R_s[j * RP + k + 1]);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const float2 xv = *reinterpret_cast<const float2*>(&x_s[(slot + SLOTS * i) * D + k]);
      acc[i] = fmaf(xv.x, r_a, fmaf(xv.y, r_b, acc[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int64_t row = r0 + slot + SLOTS * i;
    const uint32_t word = __ballot_sync(0xffffffffu, acc[i] > 0.f);
    if (lane == 0 && row < m.rows) codes[m.c_off(row) + j / 32] = word;
  }
}

// ---------------------------------------------------------------- MLP -----
// Tile of 32 rows; warp w owns rows [4w, 4w + 4).  The hidden layer is
// processed in chunks of 64 units: z = W1 x + b1 (lane l: units l, l + 32),
// h = SiLU(z), then y += W2[:, chunk] h (lane l: bits l + 32 i).  fp32 throughout.
// Small batches (queries at decode time): a cluster of 8 CTAs per 16 rows.
// CTA c computes hidden units [c hs, (c + 1) hs) of all 16 rows into its
// shared memory; after a cluster barrier every CTA copies the full hidden
// vectors out of the 8 CTAs' shared memory (distributed shared memory) and
// computes output bits [c BITS / 8, (c + 1) BITS / 8).  fp32 arithmetic as in
// the batch kernel; no global scratch and one launch.
constexpr int kMlpCluster = 8;
constexpr int kMlpClusterRows = 16;
// hidden units per CTA: a multiple of 4 so the hidden vectors move as float4
__host__ __device__ inline int mlp_rows_slice(int hidden) {
  return ((hidden + kMlpCluster - 1) / kMlpCluster + 3) & ~3;
}

// Copies n floats (n % 4 == 0, 16-byte aligned) from global memory into
// shared rows of `cols` floats at pitch `pitch`; every load of a thread is
// issued before its first shared store.
template <int U>
__device__ __forceinline__ void stage_rows(float* dst, int pitch, const float* __restrict__ src, int rows, int cols) {
  const int per_row = cols / 4, n4 = rows * per_row;
  for (int base = 0; base < n4; base += U * kThreads) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + threadIdx.x + u * kThreads;
      if (i < n4) v[u] = __ldg(reinterpret_cast<const float4*>(src) + i);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + threadIdx.x + u * kThreads;
      if (i < n4) *reinterpret_cast<float4*>(dst + (i / per_row) * pitch + (i % per_row) * 4) = v[u];
    }
  }
}

template <typename T, int BITS>
__global__ void __cluster_dims__(kMlpCluster, 1, 1) __launch_bounds__(kThreads)
mlp_rows_kernel(const T* __restrict__ x, const float* __restrict__ W1, const float* __restrict__ b1,
                const float* __restrict__ W2, const float* __restrict__ b2, int hidden, RowMap m,
                uint32_t* __restrict__ codes) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int D = kHeadDim, R = kMlpClusterRows, NB = BITS / kMlpCluster, DP = D + 4;
  // a decode step launched next on the stream may be scheduled onto free SMs
  // now; it waits for this grid to finish before it reads the codes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int rank = (int)cluster.block_rank(), tid = threadIdx.x;
  const int64_t row0 = (int64_t)(blockIdx.x / kMlpCluster) * R;
  const int hs = mlp_rows_slice(hidden), hid_pad = hs * kMlpCluster, HP = ((hidden + 3) & ~3) + 4;
  const int u0 = rank * hs, un = max(0, min(hs, hidden - u0));
  extern __shared__ __align__(16) float msm[];
  float* W1_s = msm;                  // [hs][DP]
  float* x_s = W1_s + hs * DP;        // [R][D]
  float* h_s = x_s + R * D;           // [R][hs], read by the whole cluster
  float* h_all = h_s + R * hs;        // [R][hid_pad]
  float* W2_s = h_all + R * hid_pad;  // [NB][HP]
  {
    // x rows: one 16-byte load per thread (bf16) or two (fp32), issued first
    constexpr int EPL = 16 / sizeof(T), PER_ROW = D / EPL, N = R * PER_ROW;
    uint4 raw[(N + kThreads - 1) / kThreads];
#pragma unroll
    for (int u = 0; u < (N + kThreads - 1) / kThreads; ++u) {
      const int i = tid + u * kThreads;
      const int64_t row = row0 + i / PER_ROW;
      raw[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i < N && row < m.rows) raw[u] = __ldg(reinterpret_cast<const uint4*>(x + m.x_off(row)) + i % PER_ROW);
    }
    stage_rows<8>(W1_s, DP, W1 + (int64_t)u0 * D, un, D);
    if (hidden % 4 == 0) {
      stage_rows<8>(W2_s, HP, W2 + (int64_t)(rank * NB) * hidden, NB, hidden);
    } else {
      for (int i = tid; i < NB * hidden; i += kThreads)
        W2_s[(i / hidden) * HP + i % hidden] = W2[(int64_t)(rank * NB) * hidden + i];
    }
#pragma unroll
    for (int u = 0; u < (N + kThreads - 1) / kThreads; ++u) {
      const int i = tid + u * kThreads;
      if (i >= N) continue;
      float* dst = x_s + (i / PER_ROW) * D + (i % PER_ROW) * EPL;
      if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b[e]);
          dst[2 * e] = f.x;
          dst[2 * e + 1] = f.y;
        }
      } else {
        *reinterpret_cast<uint4*>(dst) = raw[u];
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < R * hs; i += kThreads) {
    const int r = i / hs, u = i % hs;
    float h = 0.f;
    if (u < un) {
      float z = b1[u0 + u];
      const float4* w = reinterpret_cast<const float4*>(W1_s + u * DP);
      const float4* xv = reinterpret_cast<const float4*>(x_s + r * D);
#pragma unroll 8
      for (int k = 0; k < D / 4; ++k) {
        const float4 a = w[k], c = xv[k];
        z = fmaf(a.x, c.x, fmaf(a.y, c.y, fmaf(a.z, c.z, fmaf(a.w, c.w, z))));
      }
      h = z / (1.f + expf(-z));
    }
    h_s[i] = h;
  }
  cluster.sync();
  {
    // hidden vectors of all 16 rows from the 8 CTAs (hs % 4 == 0: float4 moves)
    const int n4 = R * hs / 4;
    for (int base = 0; base < n4; base += kThreads) {
      float4 v[kMlpCluster];
      const int i = base + tid;
#pragma unroll
      for (int c = 0; c < kMlpCluster; ++c)
        if (i < n4) v[c] = reinterpret_cast<const float4*>(cluster.map_shared_rank(h_s, c))[i];
#pragma unroll
      for (int c = 0; c < kMlpCluster; ++c)
        if (i < n4) *reinterpret_cast<float4*>(h_all + ((4 * i) / hs) * hid_pad + c * hs + (4 * i) % hs) = v[c];
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its h_s
  bool bit = false;
  const int r = tid / NB, j = tid % NB;
  if (tid < R * NB) {
    float y = b2[rank * NB + j];
    const float* w = W2_s + j * HP;
    const float* h = h_all + r * hid_pad;
    const int h4 = hidden & ~3;
    for (int k = 0; k < h4; k += 4) {
      const float4 a = *reinterpret_cast<const float4*>(w + k), c = *reinterpret_cast<const float4*>(h + k);
      y = fmaf(a.x, c.x, fmaf(a.y, c.y, fmaf(a.z, c.z, fmaf(a.w, c.w, y))));
    }
    for (int k = h4; k < hidden; ++k) y = fmaf(w[k], h[k], y);
    bit = y > 0.f;
  }
  const uint32_t bal = __ballot_sync(0xffffffffu, bit);
  const int64_t row = row0 + r;
  if (tid < R * NB && j == 0 && row < m.rows) {
    const int lane = tid & 31;
    if constexpr (NB == 16)
      reinterpret_cast<uint16_t*>(codes)[m.c_off(row) * 2 + rank] = (uint16_t)(bal >> lane);
    else
      reinterpret_cast<uint8_t*>(codes)[m.c_off(row) * 4 + rank] = (uint8_t)(bal >> lane);
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
mlp_encode_kernel(const T* __restrict__ x, const float* __restrict__ W1,
                  const float* __restrict__ b1, const float* __restrict__ W2,
                  const float* __restrict__ b2, int hidden, RowMap m,
                  uint32_t* __restrict__ codes) {
  constexpr int D = kHeadDim, ROWS = 32, HC = 64, TB = BITS / 32;
  constexpr int XP = ROWS + 4, W1P = HC + 1, HP = HC + 1, W2P = BITS + 1;
  extern __shared__ __align__(16) float smem[];
  float* xT = smem;               // [D][XP]
  float* W1T = xT + D * XP;       // [D][W1P]
  float* hs = W1T + D * W1P;      // [ROWS][HP]
  float* W2T = hs + ROWS * HP;    // [HC][W2P]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = (m.rows + ROWS - 1) / ROWS;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t r0 = tile * ROWS;
    __syncthreads();
    for (int i = threadIdx.x; i < ROWS * (D / 4); i += kThreads) {
      const int r = i / (D / 4), k4 = (i % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + r < m.rows) v = load4_f32(x + m.x_off(r0 + r) + k4);
      xT[(k4 + 0) * XP + r] = v.x;
      xT[(k4 + 1) * XP + r] = v.y;
      xT[(k4 + 2) * XP + r] = v.z;
      xT[(k4 + 3) * XP + r] = v.w;
    }
    float y[4][TB];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int i = 0; i < TB; ++i) y[r][i] = 0.f;
    for (int u0 = 0; u0 < hidden; u0 += HC) {
      const int hc = min(HC, hidden - u0);
      __syncthreads();
      for (int i = threadIdx.x; i < HC * D; i += kThreads) {
        const int u = i / D, k = i % D;
        W1T[k * W1P + u] = u < hc ? W1[(int64_t)(u0 + u) * D + k] : 0.f;
      }
      for (int i = threadIdx.x; i < BITS * HC; i += kThreads) {
        const int j = i / HC, u = i % HC;
        W2T[u * W2P + j] = u < hc ? W2[(int64_t)j * hidden + u0 + u] : 0.f;
      }
      __syncthreads();
      float z[4][2];
#pragma unroll
      for (int r = 0; r < 4; ++r) z[r][0] = z[r][1] = 0.f;
#pragma unroll 4
      for (int k = 0; k < D; ++k) {
        const float4 xv = *reinterpret_cast<const float4*>(&xT[k * XP + warp * 4]);
        const float wa = W1T[k * W1P + lane], wb = W1T[k * W1P + lane + 32];
        z[0][0] = fmaf(xv.x, wa, z[0][0]); z[0][1] = fmaf(xv.x, wb, z[0][1]);
        z[1][0] = fmaf(xv.y, wa, z[1][0]); z[1][1] = fmaf(xv.y, wb, z[1][1]);
        z[2][0] = fmaf(xv.z, wa, z[2][0]); z[2][1] = fmaf(xv.z, wb, z[2][1]);
        z[3][0] = fmaf(xv.w, wa, z[3][0]); z[3][1] = fmaf(xv.w, wb, z[3][1]);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int u = lane + 32 * c;
          float h = 0.f;
          if (u < hc) {
            const float zz = z[r][c] + b1[u0 + u];
            h = zz / (1.f + expf(-zz));
          }
          hs[(warp * 4 + r) * HP + u] = h;
        }
      __syncthreads();
#pragma unroll 4
      for (int u = 0; u < HC; ++u) {
        const float h0 = hs[(warp * 4 + 0) * HP + u], h1 = hs[(warp * 4 + 1) * HP + u];
        const float h2 = hs[(warp * 4 + 2) * HP + u], h3 = hs[(warp * 4 + 3) * HP + u];
#pragma unroll
        for (int i = 0; i < TB; ++i) {
          const float w = W2T[u * W2P + lane + 32 * i];
          y[0][i] = fmaf(h0, w, y[0][i]);
          y[1][i] = fmaf(h1, w, y[1][i]);
          y[2][i] = fmaf(h2, w, y[2][i]);
          y[3][i] = fmaf(h3, w, y[3][i]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int64_t row = r0 + warp * 4 + r;
#pragma unroll
      for (int i = 0; i < TB; ++i) {
        const uint32_t word = __ballot_sync(0xffffffffu, y[r][i] + b2[lane + 32 * i] > 0.f);
        if (lane == i && row < m.rows) codes[m.c_off(row) + i] = word;
      }
    }
  }
}

// --------------------------------------------------------------- SIGN -----
// Signs and fp16 L2 norm of each row.  The norm must equal the fp16 rounding
// (to nearest even) of the fp64 norm.  It is first computed in fp32: every
// square of a bf16 value is exact in fp32, so the sum of 128 of them carries a
// relative error below 128 * 2^-24 and its square root below 4e-6.  Rounding
// n (1 - 8e-6) and n (1 + 8e-6) to fp16 then gives the same value whenever the
// exact norm is far enough from an fp16 rounding midpoint, and that value is
// the exact norm's rounding; only rows whose interval straddles a midpoint
// (a few in a hundred) are summed again in fp64.  fp32 inputs (up to 24
// significant bits) always take the fp64 sum.
template <typename T>
__global__ void __launch_bounds__(kThreads)
sign_encode_kernel(const T* __restrict__ x, RowMap m, uint32_t* __restrict__ codes,
                   uint16_t* __restrict__ norms, bool vec_store) {
  // eight lanes per row, 16 dimensions per lane (bf16: two 16-byte loads,
  // fp32: four); a warp covers four rows per step and keeps kU steps of loads
  // in flight
  constexpr int D = kHeadDim, EPL = 16, V = 16 / sizeof(T), NV = EPL / V, kU = 4;
  constexpr bool kExactSquares = sizeof(T) == 2;
  const int lane = threadIdx.x & 31, sub = lane & 7, slot = lane >> 3;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  const int64_t warp_id = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  for (int64_t row0 = warp_id * 4 * kU; row0 < m.rows; row0 += warps * 4 * kU) {
    uint4 raw[kU][NV];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t row = row0 + u * 4 + slot;
#pragma unroll
      for (int v = 0; v < NV; ++v)
        raw[u][v] = row < m.rows ? __ldg(reinterpret_cast<const uint4*>(x + m.x_off(row) + sub * EPL) + v)
                                 : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t row = row0 + u * 4 + slot;
      // element i of this lane's 16 (bit operations on the loaded words, so
      // the loads stay in registers)
      auto elem = [&](int i) -> float {
        const uint4 r = raw[u][i / V];
        const int k = i % V;
        if constexpr (sizeof(T) == 2) {
          const uint32_t wd = (k >> 1) == 0 ? r.x : (k >> 1) == 1 ? r.y : (k >> 1) == 2 ? r.z : r.w;
          return __uint_as_float((k & 1) ? (wd & 0xffff0000u) : (wd << 16));
        } else {
          return __uint_as_float(k == 0 ? r.x : k == 1 ? r.y : k == 2 ? r.z : r.w);
        }
      };
      uint32_t bits = 0;
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const float f = elem(i);
        bits |= (uint32_t)(f > 0.f) << i;
        ss = fmaf(f, f, ss);
      }
      // word w = dims [32 w, 32 w + 32) = lanes 2 w (low half) and 2 w + 1
      const uint32_t hi_half = __shfl_down_sync(0xffffffffu, bits, 1);
      const uint32_t word = bits | (hi_half << 16);
      const uint32_t w1 = __shfl_down_sync(0xffffffffu, word, 2);
      const uint32_t w2 = __shfl_down_sync(0xffffffffu, word, 4);
      const uint32_t w3 = __shfl_down_sync(0xffffffffu, word, 6);
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      const float n = sqrtf(ss);
      __half h = __float2half_rn(n);
      const bool settled = kExactSquares && __half_as_ushort(__float2half_rn(n * (1.f - 8e-6f))) ==
                                                __half_as_ushort(__float2half_rn(n * (1.f + 8e-6f)));
      if (__any_sync(0xffffffffu, !settled && norms != nullptr)) {
        // some row of the warp is close to an fp16 rounding midpoint: its
        // norm from an fp64 sum (every lane of the warp takes part)
        double sd = 0.0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const double f = (double)elem(i);
          sd = fma(f, f, sd);
        }
        sd += __shfl_xor_sync(0xffffffffu, sd, 1);
        sd += __shfl_xor_sync(0xffffffffu, sd, 2);
        sd += __shfl_xor_sync(0xffffffffu, sd, 4);
        if (!settled) h = __double2half(sqrt(sd));
      }
      if (sub == 0 && row < m.rows) {
        uint32_t* dst = codes + m.c_off(row);
        if (vec_store) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(word, w1, w2, w3);
        } else {
          dst[0] = word;
          dst[1] = w1;
          dst[2] = w2;
          dst[3] = w3;
        }
        if (norms != nullptr) norms[m.n_off(row)] = __half_as_ushort(h);
      }
    }
  }
}

// ------------------------------------------------------------ row copy -----
// dst[(g * dst_group_rows + dst_row0 + t) * D + c] = src[(g * T + t) * D + c]
template <typename T>
__global__ void __launch_bounds__(kThreads)
copy_rows_kernel(const T* __restrict__ src, T* __restrict__ dst, int64_t groups, int64_t Trows,
                 int64_t dst_group_rows, int64_t dst_row0) {
  constexpr int D = kHeadDim, V = 16 / sizeof(T);
  const int64_t total = groups * Trows * (D / V);
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t row = i / (D / V), c = (i % (D / V)) * V;
    const int64_t g = row / Trows, t = row % Trows;
    const uint4 v = *reinterpret_cast<const uint4*>(src + row * D + c);
    *reinterpret_cast<uint4*>(dst + ((g * dst_group_rows + dst_row0 + t) * D + c)) = v;
  }
}

template <typename K>
int grid_for(K kernel, size_t smem, int64_t work_items) {
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  int64_t g = (int64_t)sm_count() * per_sm;
  if (work_items < g) g = work_items;
  return (int)(g < 1 ? 1 : g);
}

template <typename T, int BITS>
int run_lsh(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, cudaStream_t st) {
  if (m.rows <= kFewRows) {
    auto kernel = lsh_rows_kernel<T, BITS>;
    const size_t smem = sizeof(float) * 16 * kHeadDim + sizeof(T) * BITS * (kHeadDim + (sizeof(T) == 2 ? 2 : 1));
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "lsh rows smem attribute");
    kernel<<<(unsigned)((m.rows + 15) / 16), kThreads, smem, st>>>(static_cast<const T*>(x),
                                                                      static_cast<const T*>(h.R), m, codes);
    return cuda_check(cudaGetLastError(), "lsh rows launch");
  }
  auto kernel = lsh_encode_kernel<T, BITS>;
  const size_t smem = sizeof(float) * (kHeadDim * BITS + kHeadDim * 68);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "lsh encode smem attribute");
  const int grid = grid_for(kernel, smem, (m.rows + 63) / 64);
  kernel<<<grid, kThreads, smem, st>>>(static_cast<const T*>(x), static_cast<const T*>(h.R), m, codes);
  return cuda_check(cudaGetLastError(), "lsh encode launch");
}

// Small bf16 batches with the packed 16-bit weights: the same cluster layout
// as mlp_rows_kernel with both layers on the tensor cores (mma.sync m16n8k16;
// rows are M).  Layer 1 in bf16 with fp32 sums; h = SiLU(z) with
// sigmoid(z) = (1 + tanh(z / 2)) / 2 (hardware tanh), rounded to fp16; layer 2
// in fp16 with fp32 sums: the arithmetic of the tensor-core batch encoder.
__device__ __forceinline__ void mma16816_any(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1, bool f16) {
  if (f16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp16(void* dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ float silu_tanh(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return z * fmaf(0.5f, t, 0.5f);
}

template <int BITS>
__global__ void __cluster_dims__(kMlpCluster, 1, 1) __launch_bounds__(kThreads)
mlp_rows_tc_kernel(const __nv_bfloat16* __restrict__ x, const void* __restrict__ packed, const float* __restrict__ b1,
                   const float* __restrict__ b2, int hidden, RowMap m, uint32_t* __restrict__ codes) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int D = kHeadDim, R = kMlpClusterRows, NB = BITS / kMlpCluster, XP = D + 8;
  // a decode step launched next on the stream may be scheduled onto free SMs
  // now; it waits for this grid to finish before it reads the codes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int rank = (int)cluster.block_rank(), tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tq = lane & 3;
  const int64_t row0 = (int64_t)(blockIdx.x / kMlpCluster) * R;
  const int hp = (hidden + 63) & ~63, uc = hp / kMlpCluster, u0 = rank * uc;  // uc: multiple of 8
  const int HP = hp + 8, UP = uc + 8;
  const __nv_bfloat16* W1p = static_cast<const __nv_bfloat16*>(packed);
  const __half* W2p = reinterpret_cast<const __half*>(W1p + (size_t)hp * D);
  extern __shared__ __align__(16) unsigned char msm_raw[];
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(msm_raw);  // [R][XP]
  __nv_bfloat16* w1s = xs + R * XP;                                // [uc][XP]
  __half* hs = reinterpret_cast<__half*>(w1s + uc * XP);           // [R][UP], read by the cluster
  __half* hall = hs + R * UP;                                      // [R][HP]
  __half* w2s = hall + R * HP;                                     // [NB][HP]
  // stage x rows, this CTA's W1 rows and W2 rows with cp.async (16 bytes each)
  for (int i = tid; i < R * (D / 8); i += kThreads) {
    const int r = i / (D / 8), c = i % (D / 8);
    const int64_t row = row0 + r;
    if (row < m.rows)
      cp16(xs + r * XP + c * 8, x + m.x_off(row) + c * 8);
    else
      *reinterpret_cast<uint4*>(xs + r * XP + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int i = tid; i < uc * (D / 8); i += kThreads) {
    const int r = i / (D / 8), c = i % (D / 8);
    cp16(w1s + r * XP + c * 8, W1p + (size_t)(u0 + r) * D + c * 8);
  }
  for (int i = tid; i < NB * (hp / 8); i += kThreads) {
    const int r = i / (hp / 8), c = i % (hp / 8);
    cp16(w2s + r * HP + c * 8, W2p + (size_t)(rank * NB + r) * hp + c * 8);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // layer 1: warp w takes hidden columns [8 w', 8 w' + 8) for w' = w, w + 8, ...
  for (int nt = warp; nt < uc / 8; nt += kThreads / 32) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int k0 = ks * 16 + 2 * tq;
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(xs + gid * XP + k0);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(xs + (gid + 8) * XP + k0);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(xs + gid * XP + k0 + 8);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(xs + (gid + 8) * XP + k0 + 8);
      const uint32_t bb0 = *reinterpret_cast<const uint32_t*>(w1s + (nt * 8 + gid) * XP + k0);
      const uint32_t bb1 = *reinterpret_cast<const uint32_t*>(w1s + (nt * 8 + gid) * XP + k0 + 8);
      mma16816_any(c, a0, a1, a2, a3, bb0, bb1, false);
    }
    const int u = nt * 8 + 2 * tq;  // local hidden unit of c[0] (rows gid) and c[1]
    const float bias0 = u0 + u < hidden ? b1[u0 + u] : 0.f, bias1 = u0 + u + 1 < hidden ? b1[u0 + u + 1] : 0.f;
    *reinterpret_cast<__half2*>(hs + gid * UP + u) =
        __floats2half2_rn(silu_tanh(c[0] + bias0), silu_tanh(c[1] + bias1));
    *reinterpret_cast<__half2*>(hs + (gid + 8) * UP + u) =
        __floats2half2_rn(silu_tanh(c[2] + bias0), silu_tanh(c[3] + bias1));
  }
  cluster.sync();
  {
    // all hidden units of the 16 rows: 16-byte pieces from the 8 CTAs
    const int per_cta = R * (uc / 8);
    for (int i = tid; i < kMlpCluster * per_cta; i += kThreads) {
      const int cc = i / per_cta, j = i % per_cta, r = j / (uc / 8), c8 = j % (uc / 8);
      const __half* remote = cluster.map_shared_rank(hs, cc);
      *reinterpret_cast<uint4*>(hall + r * HP + cc * uc + c8 * 8) =
          *reinterpret_cast<const uint4*>(remote + r * UP + c8 * 8);
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its hidden units
  // layer 2: warp w < NB / 8 takes output bits [8 w, 8 w + 8) of this CTA's NB
  if (warp < NB / 8) {
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ks = 0; ks < hp / 16; ++ks) {
      const int k0 = ks * 16 + 2 * tq;
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(hall + gid * HP + k0);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(hall + (gid + 8) * HP + k0);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(hall + gid * HP + k0 + 8);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(hall + (gid + 8) * HP + k0 + 8);
      const uint32_t bb0 = *reinterpret_cast<const uint32_t*>(w2s + (warp * 8 + gid) * HP + k0);
      const uint32_t bb1 = *reinterpret_cast<const uint32_t*>(w2s + (warp * 8 + gid) * HP + k0 + 8);
      mma16816_any(c, a0, a1, a2, a3, bb0, bb1, true);
    }
    const int j = rank * NB + warp * 8 + 2 * tq;  // output bit of c[0]
    uint32_t lo = (uint32_t)(c[0] + b2[j] > 0.f) | ((uint32_t)(c[1] + b2[j + 1] > 0.f) << 1);
    uint32_t hi = (uint32_t)(c[2] + b2[j] > 0.f) | ((uint32_t)(c[3] + b2[j + 1] > 0.f) << 1);
    lo <<= 2 * tq;
    hi <<= 2 * tq;
    lo |= __shfl_xor_sync(0xffffffffu, lo, 1);
    lo |= __shfl_xor_sync(0xffffffffu, lo, 2);
    hi |= __shfl_xor_sync(0xffffffffu, hi, 1);
    hi |= __shfl_xor_sync(0xffffffffu, hi, 2);
    if (tq == 0) {
      // byte (rank * NB + 8 warp) / 8 of the row's code
      const int byte = (rank * NB) / 8 + warp;
      if (row0 + gid < m.rows) reinterpret_cast<uint8_t*>(codes)[m.c_off(row0 + gid) * 4 + byte] = (uint8_t)lo;
      if (row0 + gid + 8 < m.rows)
        reinterpret_cast<uint8_t*>(codes)[m.c_off(row0 + gid + 8) * 4 + byte] = (uint8_t)hi;
    }
  }
}

template <typename T, int BITS>
int run_mlp(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, cudaStream_t st) {
  if (m.rows <= kFewRows && sizeof(T) == 2 && h.packed != nullptr) {
    auto kernel = mlp_rows_tc_kernel<BITS>;
    const int hp = (h.hidden + 63) & ~63, uc = hp / kMlpCluster;
    const size_t smem = 2 * ((size_t)kMlpClusterRows * (kHeadDim + 8) + (size_t)uc * (kHeadDim + 8) +
                             (size_t)kMlpClusterRows * (uc + 8) + (size_t)kMlpClusterRows * (hp + 8) +
                             (size_t)(BITS / kMlpCluster) * (hp + 8));
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "mlp rows tc smem attribute");
    const int64_t clusters = (m.rows + kMlpClusterRows - 1) / kMlpClusterRows;
    kernel<<<(unsigned)(clusters * kMlpCluster), kThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(x), h.packed, h.b1, h.b2, h.hidden, m, codes);
    return cuda_check(cudaGetLastError(), "mlp rows tc launch");
  }
  if (m.rows <= kFewRows) {
    auto kernel = mlp_rows_kernel<T, BITS>;
    const int hs = mlp_rows_slice(h.hidden);
    const size_t smem = sizeof(float) * ((size_t)hs * (kHeadDim + 4) + kMlpClusterRows * kHeadDim +
                                         (size_t)kMlpClusterRows * hs + (size_t)kMlpClusterRows * hs * kMlpCluster +
                                         (size_t)(BITS / kMlpCluster) * (((h.hidden + 3) & ~3) + 4));
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_check(e, "mlp rows smem attribute");
    const int64_t clusters = (m.rows + kMlpClusterRows - 1) / kMlpClusterRows;
    kernel<<<(unsigned)(clusters * kMlpCluster), kThreads, smem, st>>>(static_cast<const T*>(x), h.W1, h.b1, h.W2,
                                                                        h.b2, h.hidden, m, codes);
    return cuda_check(cudaGetLastError(), "mlp rows launch");
  }
  auto kernel = mlp_encode_kernel<T, BITS>;
  const size_t smem = sizeof(float) * (kHeadDim * 36 + kHeadDim * 65 + 32 * 65 + 64 * (BITS + 1));
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "mlp encode smem attribute");
  const int grid = grid_for(kernel, smem, (m.rows + 31) / 32);
  kernel<<<grid, kThreads, smem, st>>>(static_cast<const T*>(x), h.W1, h.b1, h.W2, h.b2, h.hidden, m, codes);
  return cuda_check(cudaGetLastError(), "mlp encode launch");
}

template <typename T>
int run_sign(const void* x, const RowMap& m, uint32_t* codes, uint16_t* norms, cudaStream_t st) {
  auto kernel = sign_encode_kernel<T>;
  const int grid = grid_for(kernel, 0, (m.rows + 127) / 128);
  const bool vec = reinterpret_cast<uintptr_t>(codes) % 16 == 0 && m.c_row % 4 == 0 && m.c_group % 4 == 0;
  kernel<<<grid, kThreads, 0, st>>>(static_cast<const T*>(x), m, codes, norms, vec);
  return cuda_check(cudaGetLastError(), "sign encode launch");
}

}  // namespace

int launch_encode(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes,
                  uint16_t* norms, cudaStream_t st, int32_t* status) {
  if (m.rows == 0) return HKV_OK;
  if (lsh_tc_eligible(h, x, m, codes)) return launch_lsh_tc(h, x, m, codes, status, st);
  if (mlp_tc_eligible(h, x, m, codes)) return launch_mlp_tc(h, x, m, codes, status, st);
  const bool bf = h.dtype == HKV_BF16;
  switch (h.kind) {
    case HKV_HASH_LSH:
      if (h.code_bits == 128) return bf ? run_lsh<__nv_bfloat16, 128>(h, x, m, codes, st) : run_lsh<float, 128>(h, x, m, codes, st);
      return bf ? run_lsh<__nv_bfloat16, 64>(h, x, m, codes, st) : run_lsh<float, 64>(h, x, m, codes, st);
    case HKV_HASH_MLP:
      if (h.code_bits == 128) return bf ? run_mlp<__nv_bfloat16, 128>(h, x, m, codes, st) : run_mlp<float, 128>(h, x, m, codes, st);
      return bf ? run_mlp<__nv_bfloat16, 64>(h, x, m, codes, st) : run_mlp<float, 64>(h, x, m, codes, st);
    case HKV_HASH_SIGN:
      return bf ? run_sign<__nv_bfloat16>(x, m, codes, norms, st) : run_sign<float>(x, m, codes, norms, st);
  }
  return fail(HKV_ERR_INVALID_ARG, "unknown hash kind %d", h.kind);
}

int launch_copy_rows(int dtype, int64_t groups, int64_t T, const void* src, void* dst,
                     int64_t dst_group_rows, int64_t dst_row0, cudaStream_t st) {
  const int64_t items = groups * T * (dtype == HKV_BF16 ? 16 : 32);
  if (items == 0) return HKV_OK;
  int64_t grid = (items + kThreads - 1) / kThreads;
  if (grid > 4L * sm_count()) grid = 4L * sm_count();
  if (dtype == HKV_BF16)
    copy_rows_kernel<__nv_bfloat16><<<(int)grid, kThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), groups, T, dst_group_rows, dst_row0);
  else
    copy_rows_kernel<float><<<(int)grid, kThreads, 0, st>>>(
        static_cast<const float*>(src), static_cast<float*>(dst), groups, T, dst_group_rows, dst_row0);
  return cuda_check(cudaGetLastError(), "append copy launch");
}

}  // namespace hkv
