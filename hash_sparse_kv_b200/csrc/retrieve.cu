// Hamming scan + top-k selection (S4, S5), optionally fused with the query
// encoding (S2), the sparse attention over the selected and resident rows and
// the log-sum-exp merge (S6-S8): one decode step in one launch.
//
// HashEvict ("Abstract") scores cached keys by the Hamming distance between
// binarized projections of the query and of each key; Spotlight Attention
// ("Approach", "Key results") keeps the top-k keys per decode step and
// attends over them exactly, with sink and local-window tokens kept;
// RetrievalAttention ("Approach") merges partial attention results by exact
// log-sum-exp rescaling.  With grouped-query attention a KV head's score of
// token t is the sum over its g query heads:
//     D(t) = sum_h popcount(cq_h XOR ck_t)  in [0, g * bits].
//
// One launch, one block of 512 threads per SM (cooperative when a pair spans
// several blocks):
//  * The candidates of each selection unit -- a (batch, KV head) pair, or a
//    (batch, query head) pair for per-head index sets -- are cut into equal
//    contiguous segments, one per block, so no block straddles two units.
//    With a ragged batch each unit takes its window from its own length.
//  * Phase A.  Each thread streams its tokens through a private ring of
//    cp.async slots while the block encodes the query heads it needs (bf16
//    LSH on mma.sync, sign by ballots).  Per token it computes D, keeps it in
//    shared memory (uint16) and counts it in the block's histogram.
//  * Publication.  A block adds its counts up to hi = its own k-th smallest D
//    (all bins if it holds fewer than k_eff tokens) into the unit's global
//    histogram and stores its cumulative counts over [0, hi].  The threshold
//    T (smallest D whose cumulative count reaches k_eff) is at most min over
//    blocks of hi, because that block alone already has k_eff tokens at or
//    below its hi; so the global histogram is complete on [0, T].
//  * Phase B.  Wait (bounded) for all blocks of the unit, read the global
//    histogram, find T, read the lower blocks' cumulative counts at T - 1 and
//    T, then write this block's selected tokens straight to their final,
//    ascending positions in idx: tokens with D < T, and tokens with D == T in
//    ascending order until k_eff is reached.
//  * Attention.  The block attends its selected rows plus its share of the
//    unit's resident sink/local rows for all of the unit's query heads (bf16:
//    tensor-core logits and P V over 64-row tiles fetched by cp.async) and
//    writes one partial (m, l, acc).  The last g blocks of the unit to finish
//    merge one head each: M = max m_s, L = sum l_s e^{m_s - M},
//    out = sum acc_s e^{m_s - M} / L, lse = M + log L.
//  * The last block out of a unit returns its counters and histogram to zero,
//    so the workspace is ready for the next call.
//
// The group-summed distance is computed by bit-sliced arithmetic
// (hamming.cuh) instead of g * W popcounts.
#include <math.h>

#include <algorithm>
#include <mutex>

#include "hamming.cuh"
#include "internal.h"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 4;                  // cp.async groups in flight per thread
constexpr int kSlots = 2 * kGroups;         // two tokens per group
constexpr int kMaxTokensPerBlock = 65536;   // uint16 distances in shared memory (when it fits)
constexpr int kTokensPerBlockSmall = 32768; // the cap when the larger one does not fit
constexpr size_t kStaticSmem = 2048;        // bound on the kernel's static shared memory
constexpr int kMinTokensPerBlock = 2048;
constexpr int kMaxSegsPerPair = 160;        // blocks per pair (shared header buffer)
constexpr int kMaxGroup = 16;
constexpr int kQRows = 32;                  // query rows one block may encode
constexpr int kRows = 64;                   // attention tile
constexpr int kKP = kHeadDim + 4;     // K tile pitch: float4-aligned rows
constexpr int kPart = kHeadDim + 2;         // m, l, acc[128]
constexpr int kSync = 4;                    // per pair: arrivals, departures, merge ticket, merges done
constexpr int kSelCap = 2048;               // selected rows kept in shared memory
constexpr int kOut = (kMaxGroup * kHeadDim + kThreads - 1) / kThreads;

enum QEnc { kQGiven = 0, kQLsh = 1, kQSign = 2 };

struct FusedArgs {
  const uint32_t* q_codes_in;  // kQGiven: [B, Hq, W]
  uint32_t* q_codes_out;       // nullable: written by each pair's first segment
  const void* R;               // kQLsh: [bits, 128] in the dtype of q
  int qenc;
  const uint32_t* k_codes;
  int32_t* idx;
  int32_t* dist;
  const void* q;
  const void* K;
  const void* V;
  float* out;
  float* lse;
  float scale;
  int Hq, Hkv, g;
  int64_t cap, lo;
  int C, k_eff, top_k;
  int sink_n, local_start, local_n;
  int p0, nseg, per_block;
  int nbins, nbins_pad;
  uint32_t off_q, off_aq, off_sel, off_hist, off_dist;  // shared memory carve-up (bytes)
  uint32_t* sync;  // [pairs][kSync]
  uint32_t* gh;    // [pairs][nbins]: histogram of the pair (returns to zero)
  const uint32_t* next_codes;  // nullable: codes of the next call, prefetched to L2 after the scan
  int Hkv_real, unit_div;      // KV heads of the cache; selection units per KV head
  const int32_t* n_tok_b;      // nullable [B]: tokens of each sequence (ragged batch)
  int n_sink_cfg, n_local_cfg, n_max;
  uint32_t* cum;   // [pairs][nseg][nbins]: cumulative counts, window only
  float* part;     // [pairs][nseg][g][kPart]
  int32_t* status;
  uint64_t wait_ns;
  int skip_arrive;
};

// Cache row of (batch, KV head) for selection unit p (units = KV heads, or
// query heads with unit_div = g of them per KV head).
__device__ __forceinline__ int64_t kv_row(const FusedArgs& a, int p) {
  return (int64_t)(p / a.Hkv) * a.Hkv_real + (p % a.Hkv) / a.unit_div;
}


// ---- cp.async helpers (per-thread ring; each thread reads only its own slots)
template <int W>
__device__ __forceinline__ void cp_async_code(uint32_t* dst, const uint32_t* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (W == 4)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int W>
__device__ __forceinline__ void load_slot(const uint32_t* sl, uint32_t (&ck)[W]) {
  if constexpr (W == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(sl);
    ck[0] = v.x;
    ck[1] = v.y;
    ck[2] = v.z;
    ck[3] = v.w;
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(sl);
    ck[0] = v.x;
    ck[1] = v.y;
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
  // totals of the warps before this one: one load per lane and a warp sum
  uint32_t pre = lane < warp ? warp_tmp[lane] : 0u;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) pre += __shfl_xor_sync(0xffffffffu, pre, off);
  uint32_t run = x - s + pre;
  for (int i = beg; i < end; ++i) {
    run += a[i];
    a[i] = run;
  }
  __syncthreads();
}

// Exclusive prefix of v over the block's threads; *total receives the sum.
// warp_tmp: kWarps 8-byte words.
__device__ __forceinline__ uint64_t block_exclusive(uint64_t v, uint64_t* warp_tmp, uint64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  uint64_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint64_t t = warp_tmp[w];
    base += w < warp ? t : 0ull;
    tot += t;
  }
  *total = tot;
  return base + x - v;
}

// Block-wide sums of x and y; every thread receives both totals.
// warp_tmp needs 2 * kWarps words.
__device__ __forceinline__ void block_sum2(uint32_t& x, uint32_t& y, uint32_t* warp_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, off);
    y += __shfl_xor_sync(0xffffffffu, y, off);
  }
  __syncthreads();
  if (lane == 0) {
    warp_tmp[warp] = x;
    warp_tmp[kWarps + warp] = y;
  }
  __syncthreads();
  x = 0;
  y = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    x += warp_tmp[w];
    y += warp_tmp[kWarps + w];
  }
}

// Bounded wait until *ctr >= target.  Returns false on expiry.
__device__ bool wait_count(const uint32_t* ctr, uint32_t target, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; ld_acquire_gpu(ctr) < target; ++it) {
    if (globaltimer_ns() - t0 > limit_ns || it > (1u << 28)) return false;
    __nanosleep(32);
  }
  return true;
}

template <typename T>
__device__ __forceinline__ const T* tptr(const void* p) { return static_cast<const T*>(p); }

// Bring one K row and one V row (element row index `row`) into L2.
template <typename T>
__device__ __forceinline__ void prefetch_row_l2(const void* K, const void* V, int64_t row) {
  constexpr uint32_t kBytes = kHeadDim * sizeof(T);
  const T* k = tptr<T>(K) + row * kHeadDim;
  const T* v = tptr<T>(V) + row * kHeadDim;
#pragma unroll
  for (uint32_t o = 0; o < kBytes; o += 128) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(k) + o));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(v) + o));
  }
}

// Counter increments that publish the block's earlier writes (after a
// __syncthreads, a release by one thread covers the whole block's writes).
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------- attention
struct AttnSmem {
  float* q;  // [kMaxGroup][128]
  float* K;  // [kRows][kKP]
  float* V;  // [kRows][128]
  float* z;  // [kMaxGroup][kRows]
  int* tok;  // [kRows]
  float* m;
  float* l;
  float* alpha;
};

__device__ void attn_begin(int g, const AttnSmem& sm, float (&acc)[kOut]) {
#pragma unroll
  for (int j = 0; j < kOut; ++j) acc[j] = 0.f;
  if (threadIdx.x < g) {
    sm.m[threadIdx.x] = -INFINITY;
    sm.l[threadIdx.x] = 0.f;
  }
}

// 16-byte chunk of a K or V row: bf16 rows hold 8 elements per chunk, fp32 rows 4.
__device__ __forceinline__ void chunk_to_f32(const uint4& raw, float* dst, __nv_bfloat16) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&raw);
  const float2 f0 = __bfloat1622float2(b[0]), f1 = __bfloat1622float2(b[1]);
  const float2 f2 = __bfloat1622float2(b[2]), f3 = __bfloat1622float2(b[3]);
  *reinterpret_cast<float4*>(dst) = make_float4(f0.x, f0.y, f1.x, f1.y);
  *reinterpret_cast<float4*>(dst + 4) = make_float4(f2.x, f2.y, f3.x, f3.y);
}
__device__ __forceinline__ void chunk_to_f32(const uint4& raw, float* dst, float) {
  *reinterpret_cast<uint4*>(dst) = raw;
}

// Adds `nrows` rows (token row_at(i), or -1 to skip) to the online softmax,
// 64 rows per tile.  The K/V rows of tile i + 1 are loaded into registers
// while tile i is computed, so the gather latency overlaps the arithmetic.
template <typename T, typename RowAt>
__device__ void attn_rows(const FusedArgs& a, int64_t kvc, int nrows, RowAt row_at, const AttnSmem& sm,
                          float (&acc)[kOut]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = a.g;
  const T* Kp = tptr<T>(a.K) + kvc * kHeadDim;
  const T* Vp = tptr<T>(a.V) + kvc * kHeadDim;
  constexpr int EPC = 16 / sizeof(T);           // elements per 16-byte chunk
  constexpr int CPR = kHeadDim / EPC;           // chunks per row
  constexpr int kPer = kRows * CPR / kThreads;  // chunks of each matrix per thread and tile
  uint4 kr[kPer], vr[kPer];
  int tk[kPer];
  auto issue = [&](int r0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kThreads, r = i / CPR, c = i % CPR;
      tk[u] = r0 + r < nrows ? row_at(r0 + r) : -1;
      kr[u] = vr[u] = make_uint4(0u, 0u, 0u, 0u);
      if (tk[u] >= 0) {
        kr[u] = __ldg(reinterpret_cast<const uint4*>(Kp + (int64_t)tk[u] * kHeadDim) + c);
        vr[u] = __ldg(reinterpret_cast<const uint4*>(Vp + (int64_t)tk[u] * kHeadDim) + c);
      }
    }
  };
  if (nrows > 0) issue(0);
  for (int r0 = 0; r0 < nrows; r0 += kRows) {
    const int nr = min(kRows, nrows - r0);
    __syncthreads();  // the previous tile is no longer read
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kThreads, r = i / CPR, c = i % CPR;
      chunk_to_f32(kr[u], &sm.K[r * kKP + c * EPC], T());
      chunk_to_f32(vr[u], &sm.V[r * kHeadDim + c * EPC], T());
      if (c == 0) sm.tok[r] = tk[u];
    }
    __syncthreads();
    if (r0 + kRows < nrows) issue(r0 + kRows);  // in flight during this tile's arithmetic
    // logits: four lanes per (head, row), each over interleaved float4 columns
    for (int t0 = 0; t0 < g * nr * 4; t0 += kThreads) {
      const int t = t0 + tid, pr = t >> 2, qd = t & 3;
      const bool live = pr < g * nr;
      const int h = live ? pr / nr : 0, r = live ? pr % nr : 0;
      float s0 = 0.f, s1 = 0.f;
      if (live && sm.tok[r] >= 0) {
        const float* qh = sm.q + h * kHeadDim + 4 * qd;
        const float* kq = sm.K + r * kKP + 4 * qd;
#pragma unroll
        for (int i = 0; i < kHeadDim / 16; i += 2) {
          const float4 x0 = *reinterpret_cast<const float4*>(qh + 16 * i);
          const float4 y0 = *reinterpret_cast<const float4*>(kq + 16 * i);
          const float4 x1 = *reinterpret_cast<const float4*>(qh + 16 * i + 16);
          const float4 y1 = *reinterpret_cast<const float4*>(kq + 16 * i + 16);
          s0 = fmaf(x0.x, y0.x, fmaf(x0.y, y0.y, fmaf(x0.z, y0.z, fmaf(x0.w, y0.w, s0))));
          s1 = fmaf(x1.x, y1.x, fmaf(x1.y, y1.y, fmaf(x1.z, y1.z, fmaf(x1.w, y1.w, s1))));
        }
      }
      float s = s0 + s1;
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (live && qd == 0) sm.z[h * kRows + r] = sm.tok[r] >= 0 ? s * a.scale : -INFINITY;
    }
    __syncthreads();
    for (int h = warp; h < g; h += kWarps) {
      float mt = -INFINITY;
      for (int r = lane; r < nr; r += 32) mt = fmaxf(mt, sm.z[h * kRows + r]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_old = sm.m[h];
      const float m_new = fmaxf(m_old, mt);
      float ls = 0.f;
      for (int r = lane; r < nr; r += 32) {
        const float z = sm.z[h * kRows + r];
        const float e = z == -INFINITY ? 0.f : expf(z - m_new);
        sm.z[h * kRows + r] = e;
        ls += e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
      if (lane == 0) {
        const float alpha = m_new == -INFINITY ? 1.f : expf(m_old - m_new);
        sm.alpha[h] = alpha;
        sm.m[h] = m_new;
        sm.l[h] = sm.l[h] * alpha + ls;
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kOut; ++j) {
      const int o = tid + j * kThreads;
      if (o < g * kHeadDim) {
        const int h = o / kHeadDim, c = o % kHeadDim;
        const float* zh = sm.z + h * kRows;
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
        int r = 0;
        for (; r + 4 <= nr; r += 4) {
          p0 = fmaf(zh[r], sm.V[r * kHeadDim + c], p0);
          p1 = fmaf(zh[r + 1], sm.V[(r + 1) * kHeadDim + c], p1);
          p2 = fmaf(zh[r + 2], sm.V[(r + 2) * kHeadDim + c], p2);
          p3 = fmaf(zh[r + 3], sm.V[(r + 3) * kHeadDim + c], p3);
        }
        for (; r < nr; ++r) p0 = fmaf(zh[r], sm.V[r * kHeadDim + c], p0);
        acc[j] = fmaf(acc[j], sm.alpha[h], (p0 + p1) + (p2 + p3));
      }
    }
  }
}

// ---- bf16 attention on the tensor cores (mma.sync m16n8k16) ------------------
// Heads are the M dimension (g <= 16, rows >= g are zero), a 64-row tile of
// selected tokens is N for the logits and K for P V.  K/V tiles stay bf16 in
// shared memory (row pitch 272 bytes: conflict-free fragment loads) and are
// fetched with cp.async, two tiles in flight.  Logits: bf16 q and K, exact
// products, fp32 accumulation.  P V: the fp32 probabilities are split into
// bf16 hi + lo parts (two MMAs), so P keeps 16 significant bits.
constexpr int kKVPitch = kHeadDim + 8;           // bf16 elements per shared row
constexpr int kKVTile = kRows * kKVPitch * 2;    // bytes per K or V tile
constexpr int kZP = kRows + 8;                   // logit row pitch (floats)
constexpr int kPP = kRows / 2 + 4;               // probability row pitch (bf16 pairs)
constexpr int kQP = kHeadDim + 8;                // bf16 query row pitch (conflict-free fragment loads)
constexpr size_t kAttnMmaBytes = 4 * (size_t)kKVTile + sizeof(float) * kMaxGroup * kZP +
                                 2 * sizeof(uint32_t) * kMaxGroup * kPP + 2 * kMaxGroup * kQP;

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices, transposed: lane l supplies the address of row l
// (rows 8i..8i+7 form matrix i); r[i] receives the fragment of matrix i.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// Splits two fp32 values into bf16 hi and lo pairs (x ~= hi + lo).
__device__ __forceinline__ void split2(float2 x, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x.x), h1 = __float2bfloat16_rn(x.y);
  hi = pack_bf16(h0, h1);
  lo = pack_bf16(__float2bfloat16_rn(x.x - __bfloat162float(h0)), __float2bfloat16_rn(x.y - __bfloat162float(h1)));
}

// Online-softmax attention of the pair's query heads over `nrows` rows
// (token row_at(i), or -1 to skip); writes the partial (m, l, acc) of every
// head to dst[h * kPart ...].  Uses smem_attn (kAttnMmaBytes) and tok[2 * kRows].
template <typename RowAt>
__device__ void attn_mma(const FusedArgs& a, int64_t kvc, const float* aq_s, int nrows, RowAt row_at,
                         unsigned char* smem_attn, int* tok, float* m_s, float* l_s, float* alpha_s, float* dst) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = a.g;
  const int gid = lane >> 2, tq = lane & 3;
  const __nv_bfloat16* Kp = tptr<__nv_bfloat16>(a.K) + kvc * kHeadDim;
  const __nv_bfloat16* Vp = tptr<__nv_bfloat16>(a.V) + kvc * kHeadDim;
  float* z = reinterpret_cast<float*>(smem_attn + 4 * kKVTile);  // [kMaxGroup][kZP] scratch
  float* pmax = z;                                  // [8 warps][kMaxGroup] tile maxima
  float* psum = z + (kRows / 8) * kMaxGroup;        // [8 warps][kMaxGroup] tile sums
  float* m_next = z + 2 * (kRows / 8) * kMaxGroup;  // [kMaxGroup]
  // probabilities as bf16 hi and lo parts, rows of the tile in pairs: [kMaxGroup][kPP]
  uint32_t* ph = reinterpret_cast<uint32_t*>(z + kMaxGroup * kZP);
  uint32_t* pl = ph + kMaxGroup * kPP;
  for (int i = tid; i < 2 * kMaxGroup * kPP; i += kThreads) ph[i] = 0u;  // heads >= g stay zero
  // the queries as bf16 (exact: they are bf16 inputs), rows >= g zero
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(pl + kMaxGroup * kPP);  // [kMaxGroup][kQP]
  for (int i = tid; i < kMaxGroup * kHeadDim; i += kThreads) {
    const int h = i / kHeadDim, k = i % kHeadDim;
    qs[h * kQP + k] = __float2bfloat16_rn(h < g ? aq_s[h * kHeadDim + k] : 0.f);
  }
  auto kbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem_attn + (2 * b) * kKVTile); };
  auto vbuf = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem_attn + (2 * b + 1) * kKVTile); };
  constexpr int CPR = kHeadDim / 8;                 // 16-byte chunks per row
  constexpr int kPer = kRows * CPR / kThreads;      // chunks per thread per matrix
  auto issue = [&](int r0, int b) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = tid + u * kThreads, r = i / CPR, c = i % CPR;
      const int t = r0 + r < nrows ? row_at(r0 + r) : -1;
      if (c == 0) tok[b * kRows + r] = t;
      const int64_t off = (int64_t)(t >= 0 ? t : 0) * kHeadDim + c * 8;
      cp_async16_zfill(kbuf(b) + r * kKVPitch + c * 8, Kp + off, t >= 0);
      cp_async16_zfill(vbuf(b) + r * kKVPitch + c * 8, Vp + off, t >= 0);
    }
    cp_async_commit();
  };
  if (tid < g) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  float o[4] = {0.f, 0.f, 0.f, 0.f};  // P V accumulator: heads gid, gid + 8; dims 8 warp + 2 tq (+1)
  if (nrows > 0) issue(0, 0);
  for (int r0 = 0, it = 0; r0 < nrows; r0 += kRows, ++it) {
    const int b = it & 1, nr = min(kRows, nrows - r0);
    if (r0 + kRows < nrows) {
      issue(r0 + kRows, b ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* Ks = kbuf(b);
    const __nv_bfloat16* Vs = vbuf(b);
    const int* tk = tok + b * kRows;
    // logits of rows 8 w + 2 tq (+1) for heads gid and gid + 8 (warps 0..7),
    // then the tile maximum of each head through shared memory, and the
    // probabilities straight from the registers: no separate softmax pass
    float s00 = -INFINITY, s01 = -INFINITY, s10 = -INFINITY, s11 = -INFINITY;
    if (warp < kRows / 8) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const __nv_bfloat16* kr = Ks + (warp * 8 + gid) * kKVPitch + 2 * tq;
      const __nv_bfloat16* q0 = qs + gid * kQP + 2 * tq;
      const __nv_bfloat16* q1 = qs + (gid + 8) * kQP + 2 * tq;
#pragma unroll
      for (int ks = 0; ks < kHeadDim / 16; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr + ks * 16);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + ks * 16 + 8);
        const uint32_t a0 = *reinterpret_cast<const uint32_t*>(q0 + ks * 16);
        const uint32_t a1 = *reinterpret_cast<const uint32_t*>(q1 + ks * 16);
        const uint32_t a2 = *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + 8);
        const uint32_t a3 = *reinterpret_cast<const uint32_t*>(q1 + ks * 16 + 8);
        mma16816(c, a0, a1, a2, a3, b0, b1);
      }
      const int r = warp * 8 + 2 * tq;
      const bool v0 = r < nr && tk[r] >= 0, v1 = r + 1 < nr && tk[r + 1] >= 0;
      if (gid < g) {
        s00 = v0 ? c[0] * a.scale : -INFINITY;
        s01 = v1 ? c[1] * a.scale : -INFINITY;
      }
      if (gid + 8 < g) {
        s10 = v0 ? c[2] * a.scale : -INFINITY;
        s11 = v1 ? c[3] * a.scale : -INFINITY;
      }
      float mx0 = fmaxf(s00, s01), mx1 = fmaxf(s10, s11);
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      if (tq == 0) {
        pmax[warp * kMaxGroup + gid] = mx0;
        pmax[warp * kMaxGroup + gid + 8] = mx1;
      }
    }
    __syncthreads();
    if (warp < kRows / 8) {
      float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
      for (int w = 0; w < kRows / 8; ++w) {
        t0 = fmaxf(t0, pmax[w * kMaxGroup + gid]);
        t1 = fmaxf(t1, pmax[w * kMaxGroup + gid + 8]);
      }
      const float mo0 = m_s[gid < g ? gid : 0], mo1 = m_s[gid + 8 < g ? gid + 8 : 0];
      const float mn0 = fmaxf(mo0, t0), mn1 = fmaxf(mo1, t1);
      const float e00 = s00 == -INFINITY ? 0.f : expf(s00 - mn0), e01 = s01 == -INFINITY ? 0.f : expf(s01 - mn0);
      const float e10 = s10 == -INFINITY ? 0.f : expf(s10 - mn1), e11 = s11 == -INFINITY ? 0.f : expf(s11 - mn1);
      const int pr = warp * 4 + tq;  // pair index of rows 8 w + 2 tq, + 1
      uint32_t hi, lo;
      if (gid < g) {
        split2(make_float2(e00, e01), hi, lo);
        ph[gid * kPP + pr] = hi;
        pl[gid * kPP + pr] = lo;
      }
      if (gid + 8 < g) {
        split2(make_float2(e10, e11), hi, lo);
        ph[(gid + 8) * kPP + pr] = hi;
        pl[(gid + 8) * kPP + pr] = lo;
      }
      float ps0 = e00 + e01, ps1 = e10 + e11;
      ps0 += __shfl_xor_sync(0xffffffffu, ps0, 1);
      ps0 += __shfl_xor_sync(0xffffffffu, ps0, 2);
      ps1 += __shfl_xor_sync(0xffffffffu, ps1, 1);
      ps1 += __shfl_xor_sync(0xffffffffu, ps1, 2);
      if (tq == 0) {
        psum[warp * kMaxGroup + gid] = ps0;
        psum[warp * kMaxGroup + gid + 8] = ps1;
        if (warp == 0) {
          m_next[gid] = mn0;
          m_next[gid + 8] = mn1;
          alpha_s[gid] = mn0 == -INFINITY ? 1.f : expf(mo0 - mn0);
          alpha_s[gid + 8] = mn1 == -INFINITY ? 1.f : expf(mo1 - mn1);
        }
      }
    }
    __syncthreads();
    if (tid < g) {
      // running (m, l) of head tid; nothing reads them again before the next tile's second barrier
      float ls = 0.f;
#pragma unroll
      for (int w = 0; w < kRows / 8; ++w) ls += psum[w * kMaxGroup + tid];
      l_s[tid] = l_s[tid] * alpha_s[tid] + ls;
      m_s[tid] = m_next[tid];
    }
    {
      // warp w: output dims [8w, 8w + 8)
      const float al0 = gid < g ? alpha_s[gid] : 1.f, al1 = gid + 8 < g ? alpha_s[gid + 8] : 1.f;
      o[0] *= al0;
      o[1] *= al0;
      o[2] *= al1;
      o[3] *= al1;
      const uint32_t vrow = static_cast<uint32_t>(__cvta_generic_to_shared(Vs)) + (uint32_t)(warp * 8 * 2);
#pragma unroll
      for (int kp = 0; kp < kRows / 32; ++kp) {
        uint32_t bv[4];  // B fragments of k-steps 2 kp and 2 kp + 1 (rows 32 kp + lane)
        ldsm_x4_trans(vrow + (uint32_t)((kp * 32 + lane) * kKVPitch * 2), bv);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = (2 * kp + half) * 8 + tq;  // pair index of rows 16 ks + 2 tq
          const uint32_t* h0 = ph + gid * kPP + c0;
          const uint32_t* h1 = ph + (gid + 8) * kPP + c0;
          const uint32_t* l0 = pl + gid * kPP + c0;
          const uint32_t* l1 = pl + (gid + 8) * kPP + c0;
          mma16816(o, h0[0], h1[0], h0[4], h1[4], bv[2 * half], bv[2 * half + 1]);
          mma16816(o, l0[0], l1[0], l0[4], l1[4], bv[2 * half], bv[2 * half + 1]);
        }
      }
    }
    __syncthreads();  // buffer b is refilled by the next iteration's issue
  }
  // partial of every head: m, l, acc[128]
  const int c0 = warp * 8 + 2 * tq;
  if (gid < g) {
    dst[gid * kPart + 2 + c0] = o[0];
    dst[gid * kPart + 2 + c0 + 1] = o[1];
  }
  if (gid + 8 < g) {
    dst[(gid + 8) * kPart + 2 + c0] = o[2];
    dst[(gid + 8) * kPart + 2 + c0 + 1] = o[3];
  }
  if (tid < g) {
    dst[tid * kPart + 0] = m_s[tid];
    dst[tid * kPart + 1] = l_s[tid];
  }
}

__device__ void attn_end(int g, const AttnSmem& sm, const float (&acc)[kOut], float* dst) {
  const int tid = threadIdx.x;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kOut; ++j) {
    const int o = tid + j * kThreads;
    if (o < g * kHeadDim) {
      const int h = o / kHeadDim, c = o % kHeadDim;
      dst[h * kPart + 2 + c] = acc[j];
      if (c == 0) {
        dst[h * kPart + 0] = sm.m[h];
        dst[h * kPart + 1] = sm.l[h];
      }
    }
  }
}

// Merge head h of pair p over its nseg partials into out / lse.  Thread t
// takes column t % 128 of the partials s = t / 128 (mod 4) and folds them
// into a running (M, L, O) by log-sum-exp rescaling; all loads of a batch are
// issued before any is used.  The four column groups are then combined.
// red_s: 3 * kThreads floats of shared scratch.
__device__ void merge_head(const FusedArgs& a, int p, int nseg, int h, float* red_s) {
  constexpr int kQ = kThreads / kHeadDim, kB = 16;
  const int tid = threadIdx.x, g = a.g, c = tid % kHeadDim, q = tid / kHeadDim;
  const float* parts = a.part + (int64_t)p * nseg * g * kPart;
  float M = -INFINITY, L = 0.f, O = 0.f;
  for (int s0 = q; s0 < nseg; s0 += kB * kQ) {
    float2 ml[kB];
    float x[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int s = s0 + u * kQ;
      ml[u] = make_float2(-INFINITY, 0.f);
      x[u] = 0.f;
      if (s < nseg) {
        const float* src = parts + ((int64_t)s * g + h) * kPart;
        ml[u] = __ldcg(reinterpret_cast<const float2*>(src));
        x[u] = __ldcg(src + 2 + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (ml[u].x == -INFINITY) continue;
      const float mn = fmaxf(M, ml[u].x);
      const float a1 = M == -INFINITY ? 0.f : expf(M - mn), a2 = expf(ml[u].x - mn);
      L = fmaf(L, a1, ml[u].y * a2);
      O = fmaf(O, a1, x[u] * a2);
      M = mn;
    }
  }
  red_s[tid] = M;
  red_s[kThreads + tid] = L;
  red_s[2 * kThreads + tid] = O;
  __syncthreads();
  if (tid < kHeadDim) {
    float Mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kQ; ++j) Mt = fmaxf(Mt, red_s[j * kHeadDim + tid]);
    float Lt = 0.f, Ot = 0.f;
    if (Mt != -INFINITY) {
#pragma unroll
      for (int j = 0; j < kQ; ++j) {
        const float mj = red_s[j * kHeadDim + tid];
        const float w = mj == -INFINITY ? 0.f : expf(mj - Mt);
        Lt = fmaf(red_s[kThreads + j * kHeadDim + tid], w, Lt);
        Ot = fmaf(red_s[2 * kThreads + j * kHeadDim + tid], w, Ot);
      }
    }
    const int b = p / a.Hkv, kvh = p % a.Hkv;
    const int64_t orow = (int64_t)b * a.Hq + (int64_t)kvh * g + h;
    a.out[orow * kHeadDim + tid] = Lt > 0.f ? Ot / Lt : 0.f;
    if (tid == 0 && a.lse != nullptr) a.lse[orow] = Lt > 0.f ? Mt + logf(Lt) : -INFINITY;
  }
  __syncthreads();
}

// ------------------------------------------------- query encoding (in kernel)
// The block's g query heads are encoded into qc_s[h * W + w] (h < g).
// bf16 LSH: one m16n8k16 tensor-core tile per (16 rows, 8 bits, 16 dims):
// products of bf16 values are exact and accumulate in fp32.  Warp w owns bits
// [8w, 8w + 8); each lane packs its two sign bits and a 4-lane OR builds one
// byte of a row's code (bit n of the code = bit n % 8 of byte n / 8).
template <int W>
struct ProjLoads {
  static constexpr int kRV = W * 32 * (kHeadDim / 8) / kThreads;
  static constexpr int kXV = kQRows * (kHeadDim / 8) / kThreads;
  uint4 rv[kRV], xv[kXV];
};

// Global loads of R and the query rows into registers (issued early).
template <int W>
__device__ __forceinline__ void project_bf16_issue(const __nv_bfloat16* x0, int64_t x_stride, int rows,
                                                   const __nv_bfloat16* R, ProjLoads<W>& L) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int u = 0; u < ProjLoads<W>::kRV; ++u) {
    const int i = tid + u * kThreads, n = i / (kHeadDim / 8), c = (i % (kHeadDim / 8)) * 8;
    L.rv[u] = *reinterpret_cast<const uint4*>(R + (int64_t)n * kHeadDim + c);
  }
#pragma unroll
  for (int u = 0; u < ProjLoads<W>::kXV; ++u) {
    const int i = tid + u * kThreads, r = i / (kHeadDim / 8), c = (i % (kHeadDim / 8)) * 8;
    L.xv[u] = r < rows ? *reinterpret_cast<const uint4*>(x0 + (int64_t)r * x_stride + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int W>
__device__ void project_bf16_mma(const ProjLoads<W>& L, int rows, unsigned char* qbuf, uint32_t* qc_s) {
  constexpr int BITS = W * 32, XP = kHeadDim + 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __nv_bfloat16* xq = reinterpret_cast<__nv_bfloat16*>(qbuf);  // [kQRows][XP]
  __nv_bfloat16* Rq = xq + kQRows * XP;                         // [BITS][XP]
  unsigned char* qbytes = reinterpret_cast<unsigned char*>(Rq + BITS * XP);  // [kQRows][BITS / 8]
#pragma unroll
  for (int u = 0; u < ProjLoads<W>::kRV; ++u) {
    const int i = tid + u * kThreads, n = i / (kHeadDim / 8), c = (i % (kHeadDim / 8)) * 8;
    *reinterpret_cast<uint4*>(Rq + n * XP + c) = L.rv[u];
  }
#pragma unroll
  for (int u = 0; u < ProjLoads<W>::kXV; ++u) {
    const int i = tid + u * kThreads, r = i / (kHeadDim / 8), c = (i % (kHeadDim / 8)) * 8;
    *reinterpret_cast<uint4*>(xq + r * XP + c) = L.xv[u];
  }
  __syncthreads();
  const int gid = lane >> 2, tq = lane & 3;
  if (warp < BITS / 8) {
    const int n0 = warp * 8;
    for (int m0 = 0; m0 < rows; m0 += 16) {
      float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll
      for (int k0 = 0; k0 < kHeadDim; k0 += 16) {
        const uint32_t* xa = reinterpret_cast<const uint32_t*>(xq + (m0 + gid) * XP + k0 + 2 * tq);
        const uint32_t* xb = reinterpret_cast<const uint32_t*>(xq + (m0 + gid + 8) * XP + k0 + 2 * tq);
        const uint32_t* rb = reinterpret_cast<const uint32_t*>(Rq + (n0 + gid) * XP + k0 + 2 * tq);
        const uint32_t a0 = xa[0], a1 = xb[0], a2 = xa[4], a3 = xb[4], b0 = rb[0], b1 = rb[4];
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c0), "+f"(c1), "+f"(c2), "+f"(c3)
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
      }
      uint32_t lo = ((c0 > 0.f ? 1u : 0u) | (c1 > 0.f ? 2u : 0u)) << (2 * tq);
      uint32_t hi = ((c2 > 0.f ? 1u : 0u) | (c3 > 0.f ? 2u : 0u)) << (2 * tq);
      lo |= __shfl_xor_sync(0xffffffffu, lo, 1);
      lo |= __shfl_xor_sync(0xffffffffu, lo, 2);
      hi |= __shfl_xor_sync(0xffffffffu, hi, 1);
      hi |= __shfl_xor_sync(0xffffffffu, hi, 2);
      if (tq == 0) {
        if (m0 + gid < rows) qbytes[(m0 + gid) * (BITS / 8) + warp] = (unsigned char)lo;
        if (m0 + gid + 8 < rows) qbytes[(m0 + gid + 8) * (BITS / 8) + warp] = (unsigned char)hi;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < rows * W; i += kThreads) qc_s[i] = reinterpret_cast<const uint32_t*>(qbytes)[i];
}

// fp32 LSH (exact fp32 FMA, no tensor cores): thread t owns bit t % BITS of
// rows t / BITS, t / BITS + kThreads / BITS, ...
template <int W>
__device__ void project_f32_simt(const float* x0, int64_t x_stride, int rows, const float* R, unsigned char* qbuf,
                                 uint32_t* qc_s) {
  constexpr int BITS = W * 32, RP = kHeadDim + 1, SL = kThreads / BITS;
  const int tid = threadIdx.x, lane = tid & 31;
  float* xs = reinterpret_cast<float*>(qbuf);  // [kQRows][128]
  float* Rs = xs + kQRows * kHeadDim;          // [BITS][RP]
  for (int i = tid; i < BITS * kHeadDim; i += kThreads) Rs[(i / kHeadDim) * RP + i % kHeadDim] = R[i];
  for (int i = tid; i < rows * kHeadDim; i += kThreads) xs[i] = x0[(int64_t)(i / kHeadDim) * x_stride + i % kHeadDim];
  __syncthreads();
  const int j = tid % BITS, slot = tid / BITS;
  for (int r0 = 0; r0 < rows; r0 += SL) {  // a warp shares one slot, so the ballot is converged
    const int r = r0 + slot;
    float acc = 0.f;
    if (r < rows)
      for (int k = 0; k < kHeadDim; ++k) acc = fmaf(xs[r * kHeadDim + k], Rs[j * RP + k], acc);
    const uint32_t word = __ballot_sync(0xffffffffu, acc > 0.f);
    if (lane == 0 && r < rows) qc_s[r * W + j / 32] = word;
  }
}

// ------------------------------------------------------------------ kernel
// Block b serves pair p0 + b / nseg and its candidate range
// [s0, s1) = [(b % nseg) * per_block, ...): no block straddles two pairs.
template <int W, int NP, bool ATTEND, typename T>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(FusedArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + a.off_hist);
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(smem + a.off_dist);
  int32_t* sel_s = reinterpret_cast<int32_t*>(smem + a.off_sel);
  float* aq_s = reinterpret_cast<float*>(smem + a.off_aq);  // [g][128] attention queries (fp32)
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ __align__(8) uint32_t warp_tmp[2 * kWarps];
  __shared__ int sh[8];
  __shared__ float m_s[kMaxGroup], l_s[kMaxGroup], alpha_s[kMaxGroup];
  __shared__ int tok_s[2 * kRows];

  const int tid = threadIdx.x;
  const int nseg = a.nseg;
  const int p = a.p0 + (int)blockIdx.x / nseg, seg = (int)blockIdx.x % nseg;
  const int64_t kvc = kv_row(a, p) * a.cap;  // first cache row of this unit's (batch, KV head)
  // Programmatic dependent launch.  The next kernel on this stream may be
  // launched now, so its blocks are ready to take each SM this grid leaves;
  // they wait below until this grid has finished.  Before this block touches
  // global memory, the previous kernel on the stream must have finished with
  // its writes visible (without a programmatic predecessor the wait returns
  // at once).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this pair's window: uniform, or from its sequence's own length
  int lo = a.lo, C = a.C, k_eff_p = a.k_eff, sink_n = a.sink_n, local_start = a.local_start,
      local_n = a.local_n;
  if (a.n_tok_b != nullptr) {
    int nb = a.n_tok_b[p / a.Hkv];
    if (nb < 0 || nb > a.n_max) {
      if (tid == 0 && seg == 0) report(a.status, HKV_ERR_DEVICE_RANGE);
      nb = nb < 0 ? 0 : a.n_max;
    }
    sink_n = min(a.n_sink_cfg, nb);
    local_start = max(sink_n, nb - a.n_local_cfg);
    local_n = nb - local_start;
    lo = sink_n;
    C = local_start - sink_n;
    k_eff_p = min(a.top_k, C);
  }
  const int s0 = seg * a.per_block, s1 = min(s0 + a.per_block, C);
  const int len = max(s1 - s0, 0);
  const int nt = tid < len ? (len - tid + kThreads - 1) / kThreads : 0;
  uint32_t* sync = a.sync + kSync * p;
  (void)aq_s;

  // ---------------- phase A: small loads first, then the code stream ------
  // Loads issued before the code prefetch are ahead of it in the memory queues.
  const int gw = a.g * W;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * a.g;  // first query head of the pair
  uint32_t qcode_reg = 0u;
  ProjLoads<W> pj;
  if (a.qenc == kQGiven) {
    if (tid < gw) qcode_reg = __ldg(a.q_codes_in + qrow0 * W + tid);
  } else if (a.qenc == kQLsh) {
    if constexpr (sizeof(T) == 2)
      project_bf16_issue<W>(tptr<__nv_bfloat16>(a.q) + qrow0 * kHeadDim, kHeadDim, a.g, tptr<__nv_bfloat16>(a.R), pj);
  }
  float4 aq = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ATTEND && tid < a.g * (kHeadDim / 4))
    aq = load4_f32(tptr<T>(a.q) + qrow0 * kHeadDim + (tid / (kHeadDim / 4)) * kHeadDim + (tid % (kHeadDim / 4)) * 4);
  const uint32_t* pf_ptr = a.k_codes + (kvc + lo + s0 + tid) * W;
  constexpr int64_t kStep = (int64_t)kThreads * W;
  auto slot = [&](int k) { return ring + ((size_t)(k % kSlots) * kThreads + tid) * 4; };
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    if (k < nt) cp_async_code<W>(slot(k), pf_ptr + k * kStep);
    if (k & 1) cp_async_commit();
  }
  const int R_res = sink_n + local_n;
  const int n_res = seg < R_res ? (R_res - seg + nseg - 1) / nseg : 0;
  if (ATTEND && tid < n_res) {
    // the block's resident rows go to L2 now; they are attended after the scan
    const int v = seg + tid * nseg;
    const int t = v < sink_n ? v : local_start + (v - sink_n);
    prefetch_row_l2<T>(a.K, a.V, kvc + t);
  }
  // ---------------- phase A: query codes, histogram reset -------------------
  if (ATTEND && tid < a.g * (kHeadDim / 4)) *reinterpret_cast<float4*>(&aq_s[tid * 4]) = aq;
  if (a.qenc == kQGiven) {
    if (tid < gw) qc_s[tid] = qcode_reg;
  } else if (a.qenc == kQSign) {
    const T* x0 = tptr<T>(a.q) + qrow0 * kHeadDim;
    const int lane = tid & 31, warp = tid >> 5;
    for (int r = warp; r < a.g; r += kWarps) {
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const uint32_t word = __ballot_sync(0xffffffffu, to_f32(x0[(int64_t)r * kHeadDim + lane + 32 * w]) > 0.f);
        if (lane == 0) qc_s[r * W + w] = word;
      }
    }
  } else if constexpr (sizeof(T) == 2) {
    project_bf16_mma<W>(pj, a.g, smem + a.off_q, qc_s);
  } else {
    project_f32_simt<W>(tptr<float>(a.q) + qrow0 * kHeadDim, kHeadDim, a.g, tptr<float>(a.R), smem + a.off_q, qc_s);
  }
  for (int i = tid; i < a.nbins_pad; i += kThreads) hist_s[i] = 0u;
  __syncthreads();
  if (a.q_codes_out != nullptr && seg == 0)
    for (int i = tid; i < gw; i += kThreads) a.q_codes_out[qrow0 * W + i] = qc_s[i];

  // ---------------- phase A: distances and histogram -------------------------
  {
    Planes<W, NP> planes;
    build_planes<W, NP>(qc_s, a.g, planes);
    for (int k = 0; k < nt; k += 2) {
      cp_async_wait<kGroups - 1>();
      uint32_t ck0[W], ck1[W];
      load_slot<W>(slot(k), ck0);
      const bool two = k + 1 < nt;
      if (two) load_slot<W>(slot(k + 1), ck1);
      const int D0 = token_distance<W, NP>(ck0, planes);
      const int D1 = two ? token_distance<W, NP>(ck1, planes) : 0;
      const int j0 = tid + k * kThreads;
      dist_s[j0] = (uint16_t)D0;
      atomicAdd(&hist_s[D0], 1u);
      if (two) {
        dist_s[j0 + kThreads] = (uint16_t)D1;
        atomicAdd(&hist_s[D1], 1u);
      }
      if (k + kSlots < nt) cp_async_code<W>(slot(k), pf_ptr + (k + kSlots) * kStep);
      if (k + 1 + kSlots < nt) cp_async_code<W>(slot(k + 1), pf_ptr + (k + 1 + kSlots) * kStep);
      cp_async_commit();
    }
    cp_async_wait<0>();
  }
  if (a.next_codes != nullptr && tid < 32) {
    // the next call's codes for this block's range go to L2 while this call
    // selects and attends (16-byte aligned pieces; the hint skips ragged ends)
    const uintptr_t beg = reinterpret_cast<uintptr_t>(a.next_codes + (kvc + lo + s0) * W);
    const uintptr_t end = (beg + (uintptr_t)len * W * 4) & ~(uintptr_t)15;
    constexpr uintptr_t kPiece = 16384;
    for (uintptr_t o = ((beg + 15) & ~(uintptr_t)15) + (uintptr_t)tid * kPiece; o < end; o += 32 * kPiece) {
      const uint32_t n = (uint32_t)(end - o < kPiece ? end - o : kPiece);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(o), "r"(n) : "memory");
    }
  }
  if (tid == 0) sh[1] = a.nbins;  // hi
  __syncthreads();

  // ---------------- publication -----------------------------------------------
  // The segment adds its histogram counts up to hi (its own k-th smallest D,
  // or all bins if it holds fewer than k_eff tokens) into the pair's global
  // histogram, and stores its cumulative counts over [0, hi].  The pair's
  // threshold T is at most min over segments of hi (that segment alone has
  // k_eff tokens at or below its hi), so the global histogram is complete on
  // [0, T] and every segment's cumulative counts are known at T - 1 and T.
  const uint32_t k_eff = (uint32_t)k_eff_p;
  {
    block_inclusive_scan(hist_s, a.nbins, warp_tmp);
    const bool enough = hist_s[a.nbins - 1] >= k_eff;
    for (int v = tid; v < a.nbins; v += kThreads) {
      const uint32_t prev = v > 0 ? hist_s[v - 1] : 0u;
      if (enough && hist_s[v] >= k_eff && prev < k_eff) sh[1] = v;
    }
    __syncthreads();
    // k_eff == 0 (a ragged sequence without candidates): nothing to publish
    const int hi = k_eff == 0 ? -1 : enough ? sh[1] : a.nbins - 1;
    uint32_t* cum_out = a.cum + ((int64_t)p * nseg + seg) * a.nbins;
    uint32_t* gh = a.gh + (int64_t)p * a.nbins;
    for (int v = tid; v <= hi; v += kThreads) {
      const uint32_t c = hist_s[v], prev = v > 0 ? hist_s[v - 1] : 0u;
      cum_out[v] = c;
      if (c != prev) red_add_gpu(&gh[v], c - prev);
    }
    __syncthreads();
    if (tid == 0 && !(a.skip_arrive && blockIdx.x == 0)) red_release_add(&sync[0], 1u);
  }

  // ---------------- phase B: threshold and ordered compaction ---------------
  uint32_t n_sel = 0, sel_base = 0;
  if (tid == 0) sh[2] = wait_count(&sync[0], (uint32_t)nseg, a.wait_ns) ? 1 : 0;
  __syncthreads();
  if (sh[2]) {
    {
      // the pair's histogram, all loads in flight at once
      constexpr int kGL = 5;  // ceil(2049 / kThreads): up to g * bits + 1 bins
      const uint32_t* gh = a.gh + (int64_t)p * a.nbins;
      uint32_t gv[kGL];
#pragma unroll
      for (int u = 0; u < kGL; ++u) {
        const int v = tid + u * kThreads;
        gv[u] = v < a.nbins ? __ldcg(gh + v) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kGL; ++u) {
        const int v = tid + u * kThreads;
        if (v < a.nbins) hist_s[v] = gv[u];
      }
    }
    if (tid == 0) sh[5] = a.nbins - 1;
    __syncthreads();
    block_inclusive_scan(hist_s, a.nbins, warp_tmp);
    for (int v = tid; v < a.nbins; v += kThreads)
      if (hist_s[v] >= k_eff && (v == 0 || hist_s[v - 1] < k_eff)) sh[5] = v;
    __syncthreads();
    const int thr = sh[5];
    const uint32_t below = thr > 0 ? hist_s[thr - 1] : 0u;
    // tokens of the lower segments below and at the threshold
    uint32_t seg_lt = 0, seg_le = 0;
    for (int ss = tid; ss < seg; ss += kThreads) {
      const uint32_t* c = a.cum + ((int64_t)p * nseg + ss) * a.nbins;
      seg_lt += thr > 0 ? __ldcg(c + thr - 1) : 0u;
      seg_le += __ldcg(c + thr);
    }
    block_sum2(seg_lt, seg_le, warp_tmp);
    const uint32_t lower_lt = seg_lt, lower_eq = seg_le - seg_lt;
    const uint32_t ties_needed = k_eff - below;
    const uint32_t quota = ties_needed > lower_eq ? ties_needed - lower_eq : 0u;
    sel_base = lower_lt + min(lower_eq, ties_needed);
    // thread tid owns a contiguous run of this block's distances, read 8 at a
    // time; a chunk whose smallest distance exceeds T (almost all of them,
    // since k_eff is a small fraction of the tokens) is skipped after one
    // SIMD minimum
    const int per8 = (((len + kThreads - 1) / kThreads) + 7) & ~7;
    const int r0 = min(tid * per8, len), r1 = min(r0 + per8, len);
    const int nch = (r1 - r0 + 7) >> 3;
    auto chunk_min = [](const uint4& v) {
      const uint32_t m = __vminu2(__vminu2(v.x, v.y), __vminu2(v.z, v.w));
      return min(m & 0xffffu, m >> 16);
    };
    uint32_t lt = 0, eq = 0;
    for (int c = 0; c < nch; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(dist_s + r0 + 8 * c);
      if (chunk_min(v) > (uint32_t)thr) continue;
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int Dv = (int)((wd[e >> 1] >> (16 * (e & 1))) & 0xffffu);
        if (r0 + 8 * c + e < r1) {
          lt += Dv < thr;
          eq += Dv == thr;
        }
      }
    }
    uint64_t tot;
    const uint64_t ex = block_exclusive((uint64_t)lt | ((uint64_t)eq << 32), reinterpret_cast<uint64_t*>(warp_tmp), &tot);
    const uint32_t ex_lt = (uint32_t)ex, ex_eq = (uint32_t)(ex >> 32);
    n_sel = (uint32_t)tot + min((uint32_t)(tot >> 32), quota);
    uint32_t run_eq = ex_eq, pos = ex_lt + min(ex_eq, quota);
    int32_t* idx_out = a.idx + (int64_t)p * a.top_k + sel_base;
    int32_t* dist_out = a.dist ? a.dist + (int64_t)p * a.top_k + sel_base : nullptr;
    if (lt | eq) {
      for (int c = 0; c < nch; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(dist_s + r0 + 8 * c);
        if (chunk_min(v) > (uint32_t)thr) continue;
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int Dv = (int)((wd[e >> 1] >> (16 * (e & 1))) & 0xffffu);
          const int i = r0 + 8 * c + e;
          if (i >= r1) continue;
          bool take = Dv < thr;
          if (Dv == thr) take = run_eq++ < quota;
          if (take) {
            const int tok = lo + s0 + i;
            if (sel_base + pos < k_eff) {
              idx_out[pos] = tok;
              if (dist_out) dist_out[pos] = Dv;
              if constexpr (ATTEND) {
                if (pos < (uint32_t)kSelCap) sel_s[pos] = tok;
                prefetch_row_l2<T>(a.K, a.V, kvc + tok);
              }
            } else {
              report(a.status, HKV_ERR_DEVICE_RANGE);  // unreachable when the counts agree
            }
            ++pos;
          }
        }
      }
    }
    if (sel_base + n_sel > k_eff) n_sel = k_eff > sel_base ? k_eff - sel_base : 0u;
  } else if (tid == 0) {
    report(a.status, HKV_ERR_TIMEOUT);
  }
  __syncthreads();

  if constexpr (ATTEND) {
    // ---------------- attention over selected + resident rows, partial -----
    const int ns = (int)n_sel;
    const int32_t* sel_g = a.idx + (int64_t)p * a.top_k + sel_base;
    auto row_at = [&](int i) -> int {
      if (i < ns) return i < kSelCap ? sel_s[i] : sel_g[i];
      const int v = seg + (i - ns) * nseg;
      return v < sink_n ? v : local_start + (v - sink_n);
    };
    float* dst = a.part + ((int64_t)p * nseg + seg) * a.g * kPart;
    if constexpr (sizeof(T) == 2) {
      attn_mma(a, kvc, aq_s, ns + n_res, row_at, smem, tok_s, m_s, l_s, alpha_s, dst);
    } else {
      float* attn = reinterpret_cast<float*>(smem);
      const AttnSmem sm{aq_s, attn, attn + kRows * kKP, attn + kRows * kKP + kRows * kHeadDim, tok_s, m_s, l_s, alpha_s};
      float acc[kOut];
      attn_begin(a.g, sm, acc);
      attn_rows<T>(a, kvc, ns + n_res, row_at, sm, acc);
      attn_end(a.g, sm, acc, dst);
    }
    __syncthreads();
    if (tid == 0) sh[6] = (int)atom_acq_rel_add(&sync[2], 1u);
    __syncthreads();
    // ---------------- the last g blocks of the pair merge one head each -----
    const int nm = min(a.g, nseg);
    const int mi = sh[6] - (nseg - nm);
    if (mi >= 0) {
      if (tid == 0) sh[7] = wait_count(&sync[2], (uint32_t)nseg, a.wait_ns) ? 1 : 0;
      __syncthreads();
      if (sh[7]) {
        for (int h = mi; h < a.g; h += nm) merge_head(a, p, nseg, h, reinterpret_cast<float*>(smem));
      } else if (tid == 0) {
        report(a.status, HKV_ERR_TIMEOUT);
      }
      __syncthreads();
      if (tid == 0 && atomicAdd(&sync[3], 1u) == (uint32_t)(nm - 1)) {
        sync[2] = 0u;
        sync[3] = 0u;
      }
    }
  }

  // ---------------- departure; the last block out resets the counters -------
  __syncthreads();
  if (tid == 0) sh[2] = atom_acq_rel_add(&sync[1], 1u) == (uint32_t)(nseg - 1);
  __syncthreads();
  if (sh[2]) {
    for (int i = k_eff_p + tid; i < a.top_k; i += kThreads) {
      a.idx[(int64_t)p * a.top_k + i] = -1;
      if (a.dist) a.dist[(int64_t)p * a.top_k + i] = -1;
    }
    for (int v = tid; v < a.nbins; v += kThreads) a.gh[(int64_t)p * a.nbins + v] = 0u;
    if (tid == 0) {
      sync[0] = 0u;
      sync[1] = 0u;
    }
  }
}

using KernelFn = void (*)(FusedArgs);

template <bool ATTEND, typename T>
KernelFn pick(int words, int np) {
#define HKV_PICK(WV, NPV) \
  if (words == WV && np == NPV) return fused_kernel<WV, NPV, ATTEND, T>;
  HKV_PICK(2, 1) HKV_PICK(2, 2) HKV_PICK(2, 3) HKV_PICK(2, 4) HKV_PICK(2, 5)
  HKV_PICK(4, 1) HKV_PICK(4, 2) HKV_PICK(4, 3) HKV_PICK(4, 4) HKV_PICK(4, 5)
#undef HKV_PICK
  return nullptr;
}

KernelFn pick_kernel(bool attend, int dtype, int words, int np) {
  if (!attend) return pick<false, float>(words, np);
  return dtype == HKV_BF16 ? pick<true, __nv_bfloat16>(words, np) : pick<true, float>(words, np);
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
  int g, nbins, nbins_pad, np;
  int64_t C, lo;
  int k_eff;
  int nseg, per_block, pairs_per_launch;
  bool cooperative;
  uint32_t off_q, off_aq, off_sel, off_hist, off_dist;
  size_t smem;
  size_t ws_sync, ws_gh, ws_cum, ws_part, ws_total;
};

// q_elt: 0 when the query codes are given or are signs; else the element size
// of q (the kernel stages R and the query rows in shared memory).
int make_plan(const RetrieveShape& s, bool attend, int q_elt, Plan& pl) {
  pl.g = s.Hq / s.Hkv;
  const int bits = s.words * 32;
  const Window w = window(s.N, s.n_sink, s.n_local);
  pl.C = w.C;
  pl.lo = w.sink_end;
  pl.k_eff = (int)(s.top_k < w.C ? s.top_k : w.C);
  pl.nbins = pl.g * bits + 1;
  pl.nbins_pad = (pl.nbins + 3) & ~3;
  pl.np = bit_length(pl.g);
  if (pick_kernel(attend, HKV_BF16, s.words, pl.np) == nullptr)
    return fail(HKV_ERR_UNSUPPORTED, "no scan kernel for %d-bit codes and group size %d", bits, pl.g);
  const int64_t G = sm_count();
  const int P = s.B * s.Hkv;
  const int64_t C = pl.C > 0 ? pl.C : 1;
  // blocks per pair: fill the SMs, keep blocks between kMinTokensPerBlock and
  // max_tok candidates; max_tok = kMaxTokensPerBlock when the shared memory
  // of such a block fits, else kTokensPerBlockSmall
  for (const int max_tok : {kMaxTokensPerBlock, kTokensPerBlockSmall}) {
  int64_t bpp = std::max<int64_t>(1, G / std::max(P, 1));
  bpp = std::min<int64_t>(bpp, ceil_div(C, kMinTokensPerBlock));
  bpp = std::max<int64_t>(bpp, ceil_div(C, max_tok));
  if (bpp > G || bpp + 1 > kMaxSegsPerPair)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates per sequence is too many for one launch", (long long)C);
  pl.per_block = (int)(ceil_div(ceil_div(C, bpp), 32) * 32);
  pl.nseg = (int)ceil_div(C, pl.per_block);
  pl.cooperative = pl.nseg > 1;
  pl.pairs_per_launch = pl.cooperative ? (int)std::max<int64_t>(1, G / pl.nseg) : std::max(P, 1);
  const size_t ring = (size_t)kSlots * kThreads * 16;
  const size_t attn = std::max(sizeof(float) * (kRows * kKP + kRows * kHeadDim + kMaxGroup * kRows), kAttnMmaBytes);
  size_t off = attend ? std::max(ring, attn) : ring;
  pl.off_aq = (uint32_t)off;
  if (attend) off += sizeof(float) * pl.g * kHeadDim;
  pl.off_q = (uint32_t)off;
  if (q_elt == 2) off += align_up(sizeof(uint16_t) * (kQRows + bits) * (kHeadDim + 8) + kQRows * bits / 8, 16);
  if (q_elt == 4) off += align_up(sizeof(float) * (kQRows * kHeadDim + bits * (kHeadDim + 1)), 16);
  pl.off_sel = (uint32_t)off;
  if (attend) off += sizeof(int32_t) * kSelCap;
  pl.off_hist = (uint32_t)off;
  off += sizeof(uint32_t) * 2 * (size_t)pl.nbins_pad;
  pl.off_dist = (uint32_t)off;
  off += sizeof(uint16_t) * ((size_t)pl.per_block + 16);  // vector reads may run 7 past the end
  pl.smem = align_up(off, 16);
  if (pl.smem + kStaticSmem <= (size_t)max_smem_optin() || max_tok == kTokensPerBlockSmall) break;
  }
  pl.ws_sync = align_up(sizeof(uint32_t) * kSync * P, 256);
  pl.ws_gh = align_up(sizeof(uint32_t) * (size_t)P * pl.nbins, 256);
  pl.ws_cum = align_up(sizeof(uint32_t) * (size_t)P * pl.nseg * pl.nbins, 256);
  pl.ws_part = attend ? align_up(sizeof(float) * (size_t)P * pl.nseg * pl.g * kPart, 256) : 0;
  pl.ws_total = pl.ws_sync + pl.ws_gh + pl.ws_cum + pl.ws_part;
  return HKV_OK;
}

int launch_fused(const RetrieveShape& s, bool attend, int dtype, int qenc, const void* R,
                 const uint32_t* q_codes_in, uint32_t* q_codes_out, const uint32_t* k_codes, int32_t* idx,
                 int32_t* dist, const void* q, const void* K, const void* V, float scale, float* out,
                 float* lse, void* ws, size_t ws_bytes, int32_t* status, cudaStream_t st,
                 const uint32_t* next_codes = nullptr) {
  const int P = s.B * s.Hkv;
  const int q_elt = (qenc == kQLsh) ? (dtype == HKV_BF16 ? 2 : 4) : 0;
  Plan pl;
  int rc = make_plan(s, attend, q_elt, pl);
  if (rc != HKV_OK) return rc;
  if (ws_bytes < pl.ws_total || ws == nullptr)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, pl.ws_total);
  unsigned char* base = static_cast<unsigned char*>(ws);
  const Window w = window(s.N, s.n_sink, s.n_local);
  FusedArgs a{};
  a.q_codes_in = q_codes_in;
  a.q_codes_out = q_codes_out;
  a.R = R;
  a.qenc = qenc;
  a.k_codes = k_codes;
  a.next_codes = next_codes;
  a.Hkv_real = s.kv_heads > 0 ? s.kv_heads : s.Hkv;
  a.unit_div = s.Hkv / a.Hkv_real;
  a.n_tok_b = s.n_tok_b;
  a.n_sink_cfg = s.n_sink;
  a.n_local_cfg = s.n_local;
  a.n_max = (int)s.N;
  a.idx = idx;
  a.dist = dist;
  a.q = q;
  a.K = K;
  a.V = V;
  a.out = out;
  a.lse = lse;
  a.scale = scale;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = pl.g;
  a.cap = s.cap;
  a.lo = pl.lo;
  a.C = (int)pl.C;
  a.k_eff = pl.k_eff;
  a.top_k = s.top_k;
  a.sink_n = (int)w.sink_end;
  a.local_start = (int)w.local_start;
  a.local_n = (int)(s.N - w.local_start);
  a.nseg = pl.nseg;
  a.per_block = pl.per_block;
  a.nbins = pl.nbins;
  a.nbins_pad = pl.nbins_pad;
  a.off_q = pl.off_q;
  a.off_aq = pl.off_aq;
  a.off_sel = pl.off_sel;
  a.off_hist = pl.off_hist;
  a.off_dist = pl.off_dist;
  a.sync = reinterpret_cast<uint32_t*>(base);
  a.gh = reinterpret_cast<uint32_t*>(base + pl.ws_sync);
  a.cum = reinterpret_cast<uint32_t*>(base + pl.ws_sync + pl.ws_gh);
  a.part = reinterpret_cast<float*>(base + pl.ws_sync + pl.ws_gh + pl.ws_cum);
  a.status = status;
  a.wait_ns = wait_limit_ns();
  a.skip_arrive = (debug_flags() & kDebugSkipArrive) ? 1 : 0;
  KernelFn k = pick_kernel(attend, dtype, s.words, pl.np);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
  if (e != cudaSuccess) return cuda_check(e, "fused kernel shared memory");
  for (int p0 = 0; p0 < P; p0 += pl.pairs_per_launch) {
    a.p0 = p0;
    const int np = P - p0 < pl.pairs_per_launch ? P - p0 : pl.pairs_per_launch;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(np * pl.nseg));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n_attr = 0;
    // may start while the previous kernel on the stream drains (the kernel
    // waits for it before its first global access)
    attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n_attr++].val.programmaticStreamSerializationAllowed = 1;
    if (pl.cooperative) {
      attr[n_attr].id = cudaLaunchAttributeCooperative;
      attr[n_attr++].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    rc = cuda_check(cudaLaunchKernelEx(&cfg, k, a), "scan/select launch");
    if (rc != HKV_OK) return rc;
  }
  return HKV_OK;
}

}  // namespace

size_t retrieve_ws_bytes(const RetrieveShape& s) {
  Plan pl;
  if (make_plan(s, false, 0, pl) != HKV_OK) return 0;
  return pl.ws_total;
}

size_t decode_ws_bytes(const RetrieveShape& s) {
  Plan pl;
  if (make_plan(s, true, 0, pl) != HKV_OK) return 0;
  return pl.ws_total;
}

bool decode_encodes_queries(const RetrieveShape& s, int kind, int dtype) {
  if (kind != HKV_HASH_LSH && kind != HKV_HASH_SIGN) return false;
  Plan pl;
  const int q_elt = kind == HKV_HASH_LSH ? (dtype == HKV_BF16 ? 2 : 4) : 0;
  return make_plan(s, true, q_elt, pl) == HKV_OK && pl.g <= kQRows;
}

int launch_retrieve(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                    int32_t* idx, int32_t* dist, void* ws, size_t ws_bytes, int32_t* status,
                    cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  const Window w = window(s.N, s.n_sink, s.n_local);
  if (w.C == 0) {
    int rc = cuda_check(cudaMemsetAsync(idx, 0xff, sizeof(int32_t) * (size_t)P * s.top_k, st), "idx fill");
    if (rc == HKV_OK && dist)
      rc = cuda_check(cudaMemsetAsync(dist, 0xff, sizeof(int32_t) * (size_t)P * s.top_k, st), "dist fill");
    return rc;
  }
  return launch_fused(s, false, HKV_F32, kQGiven, nullptr, q_codes, nullptr, k_codes, idx, dist, nullptr,
                      nullptr, nullptr, 0.f, nullptr, nullptr, ws, ws_bytes, status, st);
}

// ---------------------------------------------------------------------------
// Retrieval with a fixed, library-owned scratch area instead of a caller
// workspace, for callers that cannot allocate device memory.  The area is a
// file-scope device array: every GPU that loads the library holds it until
// the process exits.  Host code must not pass the array's name to a kernel
// (on the host it is only a stand-in); its device address is looked up once
// per device with cudaGetSymbolAddress and cached for the life of the process
// (a cudaDeviceReset would invalidate the cached address, so the entry point
// must not be used after one).
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device.  Nothing is
// written here: each call clears, on its own stream, the part of the area
// that must start at zero, and every other part is written by the kernel
// before it is read.
int static_scratch(void** out) {
  int dev = 0;
  int rc = cuda_check(cudaGetDevice(&dev), "current device");
  if (rc != HKV_OK) return rc;
  if (dev < 0 || dev >= kMaxDevices) return fail(HKV_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    rc = cuda_check(cudaGetSymbolAddress(&p, g_static_scratch), "static scratch address");
    if (rc != HKV_OK) return rc;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return HKV_OK;
}
}  // namespace

int launch_retrieve_static(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                           int32_t* idx, int32_t* dist, int32_t* status, cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  Plan pl;
  int rc = make_plan(s, false, 0, pl);
  if (rc != HKV_OK) return rc;
  if (pl.ws_total > kStaticScratchBytes)
    return fail(HKV_ERR_CAPACITY, "this shape needs %zu bytes of scratch; the static scratch holds %zu bytes",
                pl.ws_total, kStaticScratchBytes);
  void* ws = nullptr;
  rc = static_scratch(&ws);
  if (rc != HKV_OK) return rc;
  // The counters and the pair histograms must start at zero.  A call of the
  // same shape leaves them so, but the previous call may have had another
  // shape (and so another layout of the area), or may never have run on this
  // device, so clear them every time, ordered on this call's stream.  The
  // per-block cumulative counts are written before they are read.
  rc = cuda_check(cudaMemsetAsync(ws, 0, pl.ws_sync + pl.ws_gh, st), "static scratch counters");
  if (rc != HKV_OK) return rc;
  return launch_retrieve(s, q_codes, k_codes, idx, dist, ws, kStaticScratchBytes, status, st);
}

int launch_decode(const RetrieveShape& s, int dtype, int q_kind, const void* R, const uint32_t* q_codes_in,
                  uint32_t* q_codes_out, const uint32_t* k_codes, const uint32_t* next_codes, int32_t* idx,
                  const void* q, const void* K, const void* V, float scale, float* out, float* lse, void* ws,
                  size_t ws_bytes, int32_t* status, cudaStream_t st) {
  const int qenc = q_kind == HKV_HASH_LSH ? kQLsh : q_kind == HKV_HASH_SIGN ? kQSign : kQGiven;
  return launch_fused(s, true, dtype, qenc, R, q_codes_in, q_codes_out, k_codes, idx, nullptr, q, K, V, scale,
                      out, lse, ws, ws_bytes, status, st, next_codes);
}



}  // namespace hkv
