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
//    below its hi; so the global histogram is complete on [0, T].  A unit
//    served by one block needs no exchange: T is its own hi.
//  * Speculative tile.  When a block's expected share of the selection is
//    small (many blocks per unit), it gathers, while the other blocks
//    publish, the K/V rows of its tokens with D <= tb (tb: the largest bin
//    whose cumulative count fits one tile beside its resident rows) and of
//    its share of the resident sink/local rows.  If T <= tb every selected
//    token of the block is in that tile.
//  * Phase B.  Wait (bounded) for all blocks of the unit, read the global
//    histogram, find T, read the lower blocks' cumulative counts at T - 1 and
//    T, then write this block's selected tokens straight to their final,
//    ascending positions in idx: tokens with D < T, and tokens with D == T in
//    ascending order until k_eff is reached (a mask over the speculative
//    tile, or an ordered compaction over 8-token octets of the distances).
//  * Attention.  Eight warps take 16-row steps of the block's selected and
//    resident rows, each with its own online softmax for the unit's query
//    heads on the tensor cores (logits and P V by mma.sync, P kept in
//    registers, two cp.async slots per warp), and the warps' partials are
//    merged into one block partial (m, l, acc).  The last blocks of the unit
//    to finish (up to one per 32 output columns) merge a run of the unit's
//    g * 128 output columns each: M = max m_s, L = sum l_s e^{m_s - M},
//    out = sum acc_s e^{m_s - M} / L, lse = M + log L; the last of them
//    returns the unit's counters and histogram to zero, so the workspace is
//    ready for the next call.
//
// The group-summed distance is computed by bit-sliced arithmetic
// (hamming.cuh) instead of g * W popcounts.
#include <math.h>

#include <algorithm>
#include <mutex>

#include "hamming.cuh"
#include "internal.h"
#include "normw_select.cuh"
#include "tc.cuh"

namespace hkv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kGroups = 4;                  // cp.async groups in flight per thread
constexpr int kSlots = 2 * kGroups;         // two codes per group
constexpr int kMaxTokensPerBlock = 65536;   // uint16 distances in shared memory (when it fits)
constexpr int kTokensPerBlockSmall = 32768; // the cap when the larger one does not fit
constexpr size_t kStaticSmem = 2048;        // bound on the kernel's static shared memory
constexpr int kMinTokensPerBlock = 2048;
constexpr int kMaxSegsPerPair = 160;        // blocks per pair (shared header buffer)
constexpr int kMaxGroup = 16;
constexpr int kQRows = 32;                  // query rows one block may encode
constexpr int kRows = 64;                   // attention tile
constexpr int kKP = kHeadDim + 4;     // K tile pitch: float4-aligned rows
constexpr int kPart = kHeadDim + 4;         // m, l, (2 unused), acc[128]: acc 16-byte aligned
constexpr int kSync = 4;                    // per pair: arrivals, departures, merge ticket, merges done
constexpr int kSelCap = 2048;               // selected rows kept in shared memory
constexpr int kPtCap = 2048;                // page ids of a block's scan range kept in shared memory
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
  uint32_t off_q, off_aq, off_sel, off_hist, off_dist, off_part, off_qs, off_tokw, off_pt;  // shared memory (bytes)
  int sel_cap;     // selected rows kept in shared memory
  int spec;        // load one speculative K/V tile during the threshold exchange
  uint32_t* sync;  // [pairs][kSync]
  uint32_t* gh;    // [pairs][nbins_pad]: histogram of the pair (returns to zero)
  const uint32_t* next_codes;  // nullable: codes of the next call, prefetched to L2 after the scan
  int Hkv_real, unit_div;      // KV heads of the cache; selection units per KV head
  const int32_t* n_tok_b;      // nullable [B]: tokens of each sequence (ragged batch)
  int n_sink_cfg, n_local_cfg, n_max;
  uint32_t* cum;   // [pairs][nseg][nbins_pad]: cumulative counts, window only
  float* part;     // [pairs][nseg][g][kPart]
  int32_t* status;
  uint64_t wait_ns;
  int skip_arrive;
  // paged cache (ptab != nullptr): token t of a sequence is slot t % page_size
  // of pool page ptab[b * max_pages + t / page_size]; codes, K and V are pools
  // [num_pages, Hkv_real, page_size, ...]
  const int32_t* ptab;
  int64_t max_pages, num_pages;
  int page_size, ps_shift;  // ps_shift: log2(page_size) for a power of two, else -1
};

// Cache row of (batch, KV head) for selection unit p (units = KV heads, or
// query heads with unit_div = g of them per KV head).
__device__ __forceinline__ int64_t kv_row(const FusedArgs& a, int p) {
  return (int64_t)(p / a.Hkv) * a.Hkv_real + (p % a.Hkv) / a.unit_div;
}

// The unit's row key, computed once per block: for a contiguous cache its
// first row in the code, K and V arrays; for a paged cache its batch index
// (high 32 bits) and KV head within a pool page (low 32 bits), so that the
// per-token row takes no division.
__device__ __forceinline__ int64_t unit_rows(const FusedArgs& a, int p) {
  if (a.ptab == nullptr) return kv_row(a, p) * a.cap;
  return ((int64_t)(p / a.Hkv) << 32) | (int64_t)((p % a.Hkv) / a.unit_div);
}

// Row of token t of the unit with row key kvc (unit_rows) in the code, K and
// V arrays: kvc + t for a contiguous cache; for a paged cache the row of its
// slot in its pool page, or -1 when the page id is outside the pool.
__device__ __forceinline__ int64_t cache_row(const FusedArgs& a, int /*p*/, int64_t kvc, int t) {
  if (a.ptab == nullptr) return kvc + t;
  int j, slot;
  if (a.ps_shift >= 0) {
    j = t >> a.ps_shift;
    slot = t & (a.page_size - 1);
  } else {
    j = t / a.page_size;
    slot = t - j * a.page_size;
  }
  const int pg = __ldg(a.ptab + (kvc >> 32) * a.max_pages + j);
  if (pg < 0 || (int64_t)pg >= a.num_pages) return -1;
  return ((int64_t)pg * a.Hkv_real + (kvc & 0xffffffffLL)) * a.page_size + slot;
}


#ifdef HKV_TIMELINE
// Diagnostic build only (-DHKV_TIMELINE): thread 0 of every block of the last
// fused launch records the global timer and its SM clock at each phase
// boundary, read back with hkv_debug_timeline.
constexpr int kTLBlocks = 1024, kTLStamps = 24;
__device__ unsigned long long g_hkv_tl[kTLBlocks * kTLStamps * 2];
#define HKV_TL(i)                                                                  \
  do {                                                                             \
    if (threadIdx.x == 0 && blockIdx.x < kTLBlocks) {                              \
      g_hkv_tl[(blockIdx.x * kTLStamps + (i)) * 2] = globaltimer_ns();            \
      g_hkv_tl[(blockIdx.x * kTLStamps + (i)) * 2 + 1] = (unsigned long long)clock64(); \
    }                                                                              \
  } while (0)
#else
#define HKV_TL(i) \
  do {            \
  } while (0)
#endif

// ---- cp.async helpers (attention tiles) and code loads from shared memory ---
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One code from a stage in shared memory (16- or 8-byte aligned).
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

__host__ __device__ constexpr int align_up_dev(int v, int a) { return (v + a - 1) / a * a; }

__device__ __forceinline__ uint32_t warp_incl_u32(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  return x;
}

// Exclusive prefix of v over the block's threads (thread order); *total
// receives the sum.  warp_tmp: kWarps words.  Contains two barriers.
__device__ __forceinline__ uint32_t block_excl_u32(uint32_t v, uint32_t* warp_tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t x = warp_incl_u32(v);
  __syncthreads();
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t t = warp_tmp[w];
    base += w < warp ? t : 0u;
    tot += t;
  }
  *total = tot;
  return base + x - v;
}

// Cumulative counts of the histogram h[0, nbins_pad) held four bins per
// thread: thread t owns bins [4t, 4t + 4) (h 16-byte aligned, zero past
// nbins).  cnt receives the thread's four counts, cum the cumulative count
// at each of its bins; returns the total.
__device__ __forceinline__ uint32_t hist_cum4(uint4 hv, uint32_t (&cnt)[4], uint32_t (&cum)[4], uint32_t* warp_tmp) {
  cnt[0] = hv.x;
  cnt[1] = hv.y;
  cnt[2] = hv.z;
  cnt[3] = hv.w;
  uint32_t total;
  const uint32_t ex = block_excl_u32(hv.x + hv.y + hv.z + hv.w, warp_tmp, &total);
  cum[0] = ex + cnt[0];
  cum[1] = cum[0] + cnt[1];
  cum[2] = cum[1] + cnt[2];
  cum[3] = cum[2] + cnt[3];
  return total;
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
__device__ void attn_rows(const FusedArgs& a, int p, int64_t kvc, int nrows, RowAt row_at, const AttnSmem& sm,
                          float (&acc)[kOut]) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = a.g;
  const T* Kp = tptr<T>(a.K);
  const T* Vp = tptr<T>(a.V);
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
      const int64_t row = tk[u] >= 0 ? cache_row(a, p, kvc, tk[u]) : -1;
      if (tk[u] >= 0 && row < 0) {  // a page outside the pool: the row is skipped
        if (c == 0) report(a.status, HKV_ERR_DEVICE_RANGE);
        tk[u] = -1;
      }
      if (tk[u] >= 0) {
        kr[u] = __ldg(reinterpret_cast<const uint4*>(Kp + row * kHeadDim) + c);
        vr[u] = __ldg(reinterpret_cast<const uint4*>(Vp + row * kHeadDim) + c);
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

// ---- bf16 attention on the tensor cores (mma.sync m16n8k16), split by warps --
// Each of kAW warps takes 16-row steps of the block's row list (step st =
// warp, warp + kAW, ...), with the next step's loads in flight in its second
// slot while it computes, and runs its own online softmax for the group's g heads
// (heads = M, rows >= g zero): logits S = Q K^T from ldmatrix fragments
// (bf16 q and K, exact products, fp32 sums), the running max and sum per
// head, and P V with P taken straight from the logits' accumulator layout as
// the A operand (split into bf16 hi + lo parts: 16 significant bits) and V
// fragments by ldmatrix.trans.  A step's K and V rows reach the warp's own
// shared-memory slot by cp.async; no block barrier inside the loop.  The
// warps' partials (m, l, acc) are merged once at the end (log-sum-exp
// rescaling, RetrievalAttention "Approach").
constexpr int kWR = 16;                          // rows per warp step
constexpr int kAW = 8;                           // attention warps, two slots each
constexpr int kVP = kHeadDim + 8;                // bf16 pitch of a slot row (272 bytes: conflict-free ldmatrix)
constexpr int kSlotBytes = 2 * kWR * kVP * 2;    // K rows then V rows of one step
constexpr size_t kAttnWarpBytes = (size_t)2 * kAW * kSlotBytes;
constexpr int kQP = kHeadDim + 8;                // bf16 query row pitch
// Slot k of warp w is at (k * kAW + w) * kSlotBytes, so the first slots of
// warps 0-3 (a speculative tile of kRows rows) come first; the compaction's
// octet list (at most 8192 octets: 16 KB) sits in the code ring past them.
constexpr int kCompactScratch = (kRows / kWR) * kSlotBytes;
static_assert(kCompactScratch + 2 * 8192 <= kSlots * kThreads * 16, "compaction list inside the code ring");

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


__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// The group's queries as bf16 (exact: they are bf16 inputs), rows >= g zero.
__device__ __forceinline__ void fill_qs(int g, const float* aq_s, __nv_bfloat16* qs) {
  for (int i = threadIdx.x; i < kMaxGroup * kHeadDim; i += kThreads) {
    const int h = i / kHeadDim, k = i % kHeadDim;
    qs[h * kQP + k] = __float2bfloat16_rn(h < g ? aq_s[h * kHeadDim + k] : 0.f);
  }
}

// Rows [kWR st, kWR st + kWR) of the row list (token row_at(i), or -1) into
// the calling warp's slot: lane l takes row l % 16 and half of its 16-byte
// chunks of K and V (cp.async, zero-filled for skipped rows); the tokens go
// to tokw[0, kWR).  One commit group.
template <typename RowAt>
__device__ __forceinline__ void warp_issue(const FusedArgs& a, int p, int64_t kvc, int nrows, RowAt row_at, int st,
                                           unsigned char* slot, int* tokw) {
  const int lane = threadIdx.x & 31, r = lane & 15, hf = lane >> 4;
  const int i = st * kWR + r;
  int t = i < nrows ? row_at(i) : -1;
  int64_t row = t >= 0 ? cache_row(a, p, kvc, t) : 0;
  if (row < 0) {  // a page outside the pool: the row is skipped
    if (hf == 0) report(a.status, HKV_ERR_DEVICE_RANGE);
    t = -1;
    row = 0;
  }
  if (hf == 0) tokw[r] = t;
  const __nv_bfloat16* Kp = tptr<__nv_bfloat16>(a.K) + row * kHeadDim;
  const __nv_bfloat16* Vp = tptr<__nv_bfloat16>(a.V) + row * kHeadDim;
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(slot) + r * kVP;
  __nv_bfloat16* vs = ks + kWR * kVP;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int col = (hf * 8 + c) * 8;
    cp_async16_zfill(ks + col, Kp + col, t >= 0);
    cp_async16_zfill(vs + col, Vp + col, t >= 0);
  }
  cp_async_commit();
}

// One 16-row step of the calling warp's online softmax.  m, l: running max
// and (this lane's part of the) sum of heads gid and gid + 8; o[n]: P V
// accumulator fragments of output columns [8 n, 8 n + 8).
__device__ __forceinline__ void warp_step(const unsigned char* slot, const int* tokw, const __nv_bfloat16* qs,
                                          float scale, float (&m)[2], float (&l)[2], float (&o)[16][4]) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
  const __nv_bfloat16* ks = reinterpret_cast<const __nv_bfloat16*>(slot);
  const __nv_bfloat16* vs = ks + kWR * kVP;
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: this lane addresses row mr of matrix mi
  // logits of rows [0, 8) (n-block 0) and [8, 16) (n-block 1)
  float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const uint32_t qa = smem_addr(qs + ((mi & 1) * 8 + mr) * kQP + (mi >> 1) * 8);
  const uint32_t ka0 = smem_addr(ks + mr * kVP + mi * 8);
  const uint32_t ka1 = smem_addr(ks + (8 + mr) * kVP + mi * 8);
#pragma unroll
  for (int k0 = 0; k0 < kHeadDim; k0 += 32) {
    uint32_t a0[4], a1[4], b0[4], b1[4];
    ldsm_x4(qa + 2 * k0, a0);
    ldsm_x4(qa + 2 * (k0 + 16), a1);
    ldsm_x4(ka0 + 2 * k0, b0);  // rows 0-7: k-step k0 (b0[0], b0[1]) and k0 + 16 (b0[2], b0[3])
    ldsm_x4(ka1 + 2 * k0, b1);
    mma16816(s[0], a0[0], a0[1], a0[2], a0[3], b0[0], b0[1]);
    mma16816(s[1], a0[0], a0[1], a0[2], a0[3], b1[0], b1[1]);
    mma16816(s[0], a1[0], a1[1], a1[2], a1[3], b0[2], b0[3]);
    mma16816(s[1], a1[0], a1[1], a1[2], a1[3], b1[2], b1[3]);
  }
  // rows of this lane: 2 tq, 2 tq + 1 (n-block 0), 8 + 2 tq, 9 + 2 tq (n-block 1)
  const bool v00 = tokw[2 * tq] >= 0, v01 = tokw[2 * tq + 1] >= 0;
  const bool v10 = tokw[8 + 2 * tq] >= 0, v11 = tokw[9 + 2 * tq] >= 0;
  s[0][0] = v00 ? s[0][0] * scale : -INFINITY;
  s[0][1] = v01 ? s[0][1] * scale : -INFINITY;
  s[0][2] = v00 ? s[0][2] * scale : -INFINITY;
  s[0][3] = v01 ? s[0][3] * scale : -INFINITY;
  s[1][0] = v10 ? s[1][0] * scale : -INFINITY;
  s[1][1] = v11 ? s[1][1] * scale : -INFINITY;
  s[1][2] = v10 ? s[1][2] * scale : -INFINITY;
  s[1][3] = v11 ? s[1][3] * scale : -INFINITY;
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
  const float al0 = mn0 == -INFINITY ? 1.f : expf(m[0] - mn0);
  const float al1 = mn1 == -INFINITY ? 1.f : expf(m[1] - mn1);
  auto ex = [](float z, float mx) { return z == -INFINITY ? 0.f : expf(z - mx); };
  float p[2][4];
#pragma unroll
  for (int nb = 0; nb < 2; ++nb) {
    p[nb][0] = ex(s[nb][0], mn0);
    p[nb][1] = ex(s[nb][1], mn0);
    p[nb][2] = ex(s[nb][2], mn1);
    p[nb][3] = ex(s[nb][3], mn1);
  }
  l[0] = fmaf(l[0], al0, (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]));
  l[1] = fmaf(l[1], al1, (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]));
  m[0] = mn0;
  m[1] = mn1;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    o[n][0] *= al0;
    o[n][1] *= al0;
    o[n][2] *= al1;
    o[n][3] *= al1;
  }
  // P as the A operand over the step's 16 rows: (head gid, rows 2 tq..), (gid + 8, ..),
  // (gid, 8 + 2 tq..), (gid + 8, 8 + 2 tq..)
  uint32_t ph[4], pl[4];
  split2(make_float2(p[0][0], p[0][1]), ph[0], pl[0]);
  split2(make_float2(p[0][2], p[0][3]), ph[1], pl[1]);
  split2(make_float2(p[1][0], p[1][1]), ph[2], pl[2]);
  split2(make_float2(p[1][2], p[1][3]), ph[3], pl[3]);
  const uint32_t va = smem_addr(vs + ((mi & 1) * 8 + mr) * kVP + (mi >> 1) * 8);
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // output columns [16 j, 16 j + 16)
    uint32_t bv[4];
    ldsm_x4_trans(va + 2 * 16 * j, bv);
    mma16816(o[2 * j], ph[0], ph[1], ph[2], ph[3], bv[0], bv[1]);
    mma16816(o[2 * j], pl[0], pl[1], pl[2], pl[3], bv[0], bv[1]);
    mma16816(o[2 * j + 1], ph[0], ph[1], ph[2], ph[3], bv[2], bv[3]);
    mma16816(o[2 * j + 1], pl[0], pl[1], pl[2], pl[3], bv[2], bv[3]);
  }
}

// Online-softmax attention of the pair's g query heads over `nrows` rows
// (token row_at(i), or -1 to skip); writes the partial (m, l, acc) of every
// head to dst[h * kPart ...].  slots: kAttnWarpBytes of shared memory (also
// the merge scratch at the end); tokw: kWarps * kWR ints; qs: the bf16
// queries (fill_qs).  pre: the first step of warps [0, pre_steps) was already
// issued (warp_issue with this row_at) and tokw entries may since have been
// set to -1 for rows to skip.  Starts and ends with a block barrier.
template <typename RowAt>
__device__ void attn_warps(const FusedArgs& a, int p, int64_t kvc, int nrows, RowAt row_at, unsigned char* slots, int* tokw,
                           const __nv_bfloat16* qs, float* dst, int pre_steps) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, tq = lane & 3, g = a.g;
  auto slot = [&](int k) { return slots + (size_t)(k * kAW + warp) * kSlotBytes; };
  auto tw = [&](int k) { return tokw + (k * kAW + warp) * kWR; };
  __syncthreads();  // qs and any earlier use of the slots
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  const int nsteps = (nrows + kWR - 1) / kWR;
  if (warp < kAW) {
    // step j of this warp is st = warp + j kAW, in slot j % 2
    if (warp >= pre_steps && warp < nsteps) warp_issue(a, p, kvc, nrows, row_at, warp, slot(0), tw(0));
    for (int j = 0, st = warp; st < nsteps; ++j, st += kAW) {
      const int nx = st + kAW;
      if (nx < nsteps) {
        warp_issue(a, p, kvc, nrows, row_at, nx, slot((j + 1) & 1), tw((j + 1) & 1));
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      warp_step(slot(j & 1), tw(j & 1), qs, a.scale, m, l, o);
      __syncwarp();  // slot j % 2 is refilled next
    }
  }
  HKV_TL(19);
  l[0] += __shfl_xor_sync(0xffffffffu, l[0], 1);
  l[0] += __shfl_xor_sync(0xffffffffu, l[0], 2);
  l[1] += __shfl_xor_sync(0xffffffffu, l[1], 1);
  l[1] += __shfl_xor_sync(0xffffffffu, l[1], 2);
  __syncthreads();  // every warp is done with its slots: they become the merge scratch
  float* wp = reinterpret_cast<float*>(slots);   // [kAW][g][kPart]
  float* wts = wp + (size_t)kAW * g * kPart;     // [kAW][kMaxGroup] weights
  float* ML = wts + kAW * kMaxGroup;             // [g][2]: M, L
  const int nact = min(kAW, nsteps);             // warps that took a step
  if (warp < nact) {
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      if (gid < g) *reinterpret_cast<float2*>(wp + ((size_t)warp * g + gid) * kPart + 4 + 8 * n + 2 * tq) = make_float2(o[n][0], o[n][1]);
      if (gid + 8 < g)
        *reinterpret_cast<float2*>(wp + ((size_t)warp * g + gid + 8) * kPart + 4 + 8 * n + 2 * tq) = make_float2(o[n][2], o[n][3]);
    }
    if (tq == 0) {
      if (gid < g) {
        wp[((size_t)warp * g + gid) * kPart] = m[0];
        wp[((size_t)warp * g + gid) * kPart + 1] = l[0];
      }
      if (gid + 8 < g) {
        wp[((size_t)warp * g + gid + 8) * kPart] = m[1];
        wp[((size_t)warp * g + gid + 8) * kPart + 1] = l[1];
      }
    }
  }
  __syncthreads();
  HKV_TL(20);
  if (tid < nact * g) {  // weight of warp w for head h
    const int w = tid / g, h = tid % g;
    float M = -INFINITY;
    for (int v = 0; v < nact; ++v) M = fmaxf(M, wp[((size_t)v * g + h) * kPart]);
    const float mw = wp[((size_t)w * g + h) * kPart];
    wts[w * kMaxGroup + h] = mw == -INFINITY ? 0.f : expf(mw - M);
    if (w == 0) ML[2 * h] = M;
  }
  __syncthreads();
  if (tid < g) {
    float L = 0.f;
    for (int v = 0; v < nact; ++v) L = fmaf(wp[((size_t)v * g + tid) * kPart + 1], wts[v * kMaxGroup + tid], L);
    ML[2 * tid + 1] = L;
    if (nact == 0) ML[2 * tid] = -INFINITY;  // no rows: an empty partial
  }
  for (int i = tid; i < g * kHeadDim; i += kThreads) {
    const int h = i / kHeadDim, c = i % kHeadDim;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < nact; ++w) O = fmaf(wp[((size_t)w * g + h) * kPart + 4 + c], wts[w * kMaxGroup + h], O);
    dst[h * kPart + 4 + c] = O;
  }
  __syncthreads();  // ML (L of every head) is complete
  if (tid < g) {
    dst[tid * kPart] = ML[2 * tid];
    dst[tid * kPart + 1] = ML[2 * tid + 1];
  }
  __syncthreads();
}

__device__ void attn_end(int g, const AttnSmem& sm, const float (&acc)[kOut], float* dst) {
  const int tid = threadIdx.x;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kOut; ++j) {
    const int o = tid + j * kThreads;
    if (o < g * kHeadDim) {
      const int h = o / kHeadDim, c = o % kHeadDim;
      dst[h * kPart + 4 + c] = acc[j];
      if (c == 0) {
        dst[h * kPart + 0] = sm.m[h];
        dst[h * kPart + 1] = sm.l[h];
      }
    }
  }
}

// Merge of the pair's output columns [col0, col0 + ncols) (column c is
// dimension c % 128 of query head c / 128 of the group; ncols <= kThreads
// and a multiple of 32) from its nseg partials (RetrievalAttention,
// "Approach": exact log-sum-exp rescaling):
//   M = max_s m_s,  w_s = e^{m_s - M},  L = sum_s l_s w_s,
//   out = sum_s acc_s w_s / L,  lse = M + log L.
// Warp w computes M, the weights and L of the range's w-th head while every
// thread has its first batch of accumulators in flight (thread (c, q):
// column c, segments q, q + Q, ... with Q = kThreads / ncols); a shared
// reduction over q finishes each column; the thread of a head's column 0
// writes its lse.  scratch: 5 * nseg + kThreads + 10 floats.
__device__ __noinline__ void merge_cols(const float* part, float* out, float* lse, int Hq, int Hkv, int g, int p,
                                        int nseg, int col0, int ncols, float* scratch) {
  constexpr int kB = 10;  // segments per thread and batch
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Q = kThreads / ncols, h0 = col0 / kHeadDim, nh = (col0 + ncols - 1) / kHeadDim - h0 + 1;
  float* w_s = scratch;                   // [nh][nseg]
  float* red_s = scratch + 5 * nseg;      // [Q][ncols]
  float* ML_s = red_s + kThreads;         // [nh][2]
  const float* base = part + (int64_t)p * nseg * g * kPart;
  const int64_t sstride = (int64_t)g * kPart;
  const bool act = tid < Q * ncols;
  const int cc = col0 + tid % ncols, q = tid / ncols, h = cc / kHeadDim, c = cc % kHeadDim;
  const float* pc = base + (int64_t)h * kPart + 4 + c;
  float x[kB];
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int sg = q + u * Q;
    x[u] = act && sg < nseg ? __ldcg(pc + sg * sstride) : 0.f;
  }
  if (warp < nh) {
    // one round of loads: every (m, l) of the head in registers
    const float* ph = base + (int64_t)(h0 + warp) * kPart;
    float2 ml[(kMaxSegsPerPair + 31) / 32];
    float M = -INFINITY;
#pragma unroll
    for (int u = 0; u < (kMaxSegsPerPair + 31) / 32; ++u) {
      const int sg = lane + 32 * u;
      ml[u] = sg < nseg ? __ldcg(reinterpret_cast<const float2*>(ph + sg * sstride)) : make_float2(-INFINITY, 0.f);
      M = fmaxf(M, ml[u].x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
#pragma unroll
    for (int u = 0; u < (kMaxSegsPerPair + 31) / 32; ++u) {
      const int sg = lane + 32 * u;
      const float w = ml[u].x == -INFINITY ? 0.f : expf(ml[u].x - M);
      if (sg < nseg) w_s[warp * nseg + sg] = w;
      L = fmaf(ml[u].y, w, L);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) {
      ML_s[2 * warp] = M;
      ML_s[2 * warp + 1] = L;
    }
  }
  __syncthreads();
  const float* wh = w_s + (h - h0) * nseg;
  float o = 0.f;
  for (int s0 = q;; s0 += kB * Q) {
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int sg = s0 + u * Q;
      if (act && sg < nseg) o = fmaf(x[u], wh[sg], o);
    }
    if (s0 + kB * Q >= nseg) break;
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int sg = s0 + kB * Q + u * Q;
      x[u] = act && sg < nseg ? __ldcg(pc + sg * sstride) : 0.f;
    }
  }
  if (act) red_s[q * ncols + tid % ncols] = o;
  __syncthreads();
  if (tid < ncols) {
    float O = 0.f;
    for (int k = 0; k < Q; ++k) O += red_s[k * ncols + tid];
    const float M = ML_s[2 * (h - h0)], L = ML_s[2 * (h - h0) + 1];
    const int b = p / Hkv, kvh = p % Hkv;
    const int64_t orow = (int64_t)b * Hq + (int64_t)kvh * g + h;
    out[orow * kHeadDim + c] = L > 0.f ? O / L : 0.f;
    if (c == 0 && lse != nullptr) lse[orow] = L > 0.f ? M + logf(L) : -INFINITY;
  }
  __syncthreads();
}

// merge_cols for one run of 32 columns [32 j, 32 j + 32) (inside head j / 4),
// with the segment groups fixed at compile time: thread (c, q) sums column
// c over segments q, q + 16, ... (one round of loads for up to 160
// segments).  scratch: nseg + 16 * 32 + 2 floats.
__device__ __noinline__ void merge_slice(const float* part, float* out, float* lse, int Hq, int Hkv, int g, int p,
                                         int nseg, int j, float* scratch) {
  constexpr int kQ = kThreads / 32;                     // segment groups
  constexpr int kB = (kMaxSegsPerPair + kQ - 1) / kQ;  // segments per thread
  const int tid = threadIdx.x, lane = tid & 31, q = tid >> 5, h = j >> 2, c = ((j & 3) << 5) + lane;
  float* w_s = scratch;           // [nseg]
  float* red_s = scratch + nseg;  // [kQ][32]
  float* ML_s = red_s + kQ * 32;  // M, L
  const float* parts = part + (int64_t)p * nseg * g * kPart + (int64_t)h * kPart;
  const int64_t sstride = (int64_t)g * kPart;
  float x[kB];
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int sg = q + u * kQ;
    x[u] = sg < nseg ? __ldcg(parts + sg * sstride + 4 + c) : 0.f;
  }
  if (tid < 32) {
    float M = -INFINITY;
    float2 ml[(kMaxSegsPerPair + 31) / 32];
#pragma unroll
    for (int u = 0; u < (kMaxSegsPerPair + 31) / 32; ++u) {
      const int sg = lane + 32 * u;
      ml[u] = sg < nseg ? __ldcg(reinterpret_cast<const float2*>(parts + sg * sstride)) : make_float2(-INFINITY, 0.f);
      M = fmaxf(M, ml[u].x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
#pragma unroll
    for (int u = 0; u < (kMaxSegsPerPair + 31) / 32; ++u) {
      const int sg = lane + 32 * u;
      const float w = ml[u].x == -INFINITY ? 0.f : expf(ml[u].x - M);
      if (sg < nseg) w_s[sg] = w;
      L = fmaf(ml[u].y, w, L);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) {
      ML_s[0] = M;
      ML_s[1] = L;
    }
  }
  __syncthreads();
  float o = 0.f;
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int sg = q + u * kQ;
    if (sg < nseg) o = fmaf(x[u], w_s[sg], o);
  }
  red_s[q * 32 + lane] = o;
  __syncthreads();
  if (tid < 32) {
    float O = 0.f;
#pragma unroll
    for (int k = 0; k < kQ; ++k) O += red_s[k * 32 + lane];
    const float M = ML_s[0], L = ML_s[1];
    const int b = p / Hkv, kvh = p % Hkv;
    const int64_t orow = (int64_t)b * Hq + (int64_t)kvh * g + h;
    out[orow * kHeadDim + c] = L > 0.f ? O / L : 0.f;
    if (c == 0 && lse != nullptr) lse[orow] = L > 0.f ? M + logf(L) : -INFINITY;
  }
  __syncthreads();
}

// The merging blocks of a pair and the columns each takes: the last nm of
// its nseg blocks, each one run of ncols columns (a multiple of 32, at
// least 32), so that every block's share is one pass of merge_cols.
struct MergeSplit {
  int nm, ncols;
};
__device__ __forceinline__ MergeSplit merge_split(int g, int nseg) {
  const int cols = g * kHeadDim;
  const int nm = min(nseg, cols / 32);
  const int per = (cols + nm - 1) / nm;
  return MergeSplit{nm, min(((per + 31) / 32) * 32, kThreads)};
}

// Block mi (of the nm merging blocks) merges columns [mi * ncols, ...) of
// the pair, in pieces of at most kThreads.
__device__ __forceinline__ void merge_share(const float* part, float* out, float* lse, int Hq, int Hkv, int g, int p,
                                            int nseg, int mi, MergeSplit ms, float* scratch) {
  const int cols = g * kHeadDim;
  for (int c0 = mi * ms.ncols; c0 < cols; c0 += ms.nm * ms.ncols) {
    if (ms.ncols == 32)
      merge_slice(part, out, lse, Hq, Hkv, g, p, nseg, c0 / 32, scratch);
    else
      merge_cols(part, out, lse, Hq, Hkv, g, p, nseg, c0, min(ms.ncols, cols - c0), scratch);
  }
}

// out / lse of every query head of pair p from the block's own partial (one
// block per pair): out = acc / l, lse = m + log l.
__device__ void finish_single(const FusedArgs& a, int p, const float* part_s) {
  const int g = a.g;
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  for (int o = threadIdx.x; o < g * 32; o += kThreads) {
    const int h = o >> 5, c4 = o & 31;
    const float* src = part_s + h * kPart;
    const float l = src[1];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float4 x = reinterpret_cast<const float4*>(src + 4)[c4];
    const int64_t orow = (int64_t)b * a.Hq + (int64_t)kvh * g + h;
    *reinterpret_cast<float4*>(a.out + orow * kHeadDim + 4 * c4) = make_float4(x.x * inv, x.y * inv, x.z * inv, x.w * inv);
    if (c4 == 0 && a.lse != nullptr) a.lse[orow] = l > 0.f ? src[0] + logf(l) : -INFINITY;
  }
}

// Exclusive prefix over the warp's lanes of a per-lane count x in [0, 16),
// and its warp total, from one ballot per bit (no shuffle chain).
__device__ __forceinline__ void warp_prefix4(uint32_t x, uint32_t& excl, uint32_t& total) {
  const uint32_t lt = lanemask_lt();
  excl = total = 0u;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t m = __ballot_sync(0xffffffffu, (x >> b) & 1u);
    excl += (uint32_t)__popc(m & lt) << b;
    total += (uint32_t)__popc(m) << b;
  }
}

// Ordered compaction of the block's distances dist_s[0, len): emits, in
// ascending index order, every i with D < thr and the first `quota` with
// D == thr, as emit(pos, i, D) with pos the rank among the emitted ones;
// returns their number.  The unit of work is an octet: 8 consecutive
// distances, one 16-byte load.
//  1. thread t takes a contiguous run of octets (read in a rotated order, so
//     a warp's loads hit distinct banks) and flags those whose smallest
//     distance is <= thr; one block prefix lists the flagged octets in
//     ascending order;
//  2. warp w takes a contiguous run of listed octets, 32 at a time (one per
//     lane), and sums the lanes' counts below and at thr;
//  3. the warps' totals give each warp its base, and the warps emit their
//     octets' tokens, ranked by ballot prefix sums of the per-lane counts.
// scratch: 2 bytes per octet of shared memory; dist_s readable 8 entries past
// len.  All threads call it (four barriers).
template <typename Emit>
__device__ uint32_t compact_block(const uint16_t* dist_s, int len, int thr, uint32_t quota, uint32_t* warp_tmp,
                                  unsigned char* scratch, Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int noct = (len + 7) >> 3;
  uint16_t* olist = reinterpret_cast<uint16_t*>(scratch);  // [noct]
  const uint32_t t = (uint32_t)thr;
  auto oct_min = [](const uint4& v) {
    const uint32_t m = __vminu2(__vminu2(v.x, v.y), __vminu2(v.z, v.w));
    return min(m & 0xffffu, m >> 16);
  };
  // counts below and at thr among the octet's tokens [8 o, 8 o + 8) that are < len
  auto count8 = [&](const uint4& v, int o, uint32_t& lt, uint32_t& eq) {
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
    lt = eq = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t D = (wd[e >> 1] >> (16 * (e & 1))) & 0xffffu;
      const bool in = 8 * o + e < len;
      lt += (in && D < t) ? 1u : 0u;
      eq += (in && D == t) ? 1u : 0u;
    }
  };
  // 1. listed octets
  int R = 1;  // octets per thread: a power of two (<= 16 for 65536 tokens)
  while (R * kThreads < noct) R <<= 1;
  const int o0 = tid * R;
  uint32_t fl = 0, nf = 0;
  for (int j = 0; j < R; ++j) {
    const int r = (j + tid) & (R - 1), o = o0 + r;
    if (o < noct && oct_min(*reinterpret_cast<const uint4*>(dist_s + 8 * o)) <= t) {
      fl |= 1u << r;
      ++nf;
    }
  }
  uint32_t nlist;
  uint32_t pos = block_excl_u32(nf, warp_tmp, &nlist);
  for (int r = 0; r < R; ++r)
    if ((fl >> r) & 1u) olist[pos++] = (uint16_t)(o0 + r);
  __syncthreads();
  HKV_TL(16);
  // 2. counts of each warp's run of listed octets
  const int per = ((int)nlist + kWarps - 1) / kWarps;
  const int f0 = min(warp * per, (int)nlist), f1 = min(f0 + per, (int)nlist);
  uint32_t wl = 0, we = 0;
  for (int f = f0 + lane; f < f1; f += 32) {
    const int o = olist[f];
    uint32_t lt, eq;
    count8(*reinterpret_cast<const uint4*>(dist_s + 8 * o), o, lt, eq);
    wl += lt;
    we += eq;
  }
  wl = __reduce_add_sync(0xffffffffu, wl);
  we = __reduce_add_sync(0xffffffffu, we);
  if (lane == 0) {
    warp_tmp[kWarps + warp] = wl;
    warp_tmp[2 * kWarps + warp] = we;
  }
  __syncthreads();
  HKV_TL(17);
  uint32_t run_lt = 0, run_eq = 0, tot_lt = 0, tot_eq = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = warp_tmp[kWarps + w], y = warp_tmp[2 * kWarps + w];
    run_lt += w < warp ? x : 0u;
    run_eq += w < warp ? y : 0u;
    tot_lt += x;
    tot_eq += y;
  }
  HKV_TL(18);
  // 3. emit
  for (int fb = f0; fb < f1; fb += 32) {
    const int f = fb + lane;
    const bool live = f < f1;
    const int o = live ? olist[f] : 0;
    const uint4 v = live ? *reinterpret_cast<const uint4*>(dist_s + 8 * o) : make_uint4(~0u, ~0u, ~0u, ~0u);
    uint32_t lt, eq;
    count8(v, o, lt, eq);
    if (!live) lt = eq = 0u;
    uint32_t ex_lt, ex_eq, row_lt, row_eq;
    warp_prefix4(lt, ex_lt, row_lt);
    warp_prefix4(eq, ex_eq, row_eq);
    if (lt | eq) {
      uint32_t bl = run_lt + ex_lt, be = run_eq + ex_eq;
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t D = (wd[e >> 1] >> (16 * (e & 1))) & 0xffffu;
        const int i = 8 * o + e;
        if (i >= len) continue;
        if (D < t) {
          emit(bl + min(be, quota), i, (int)D);
          ++bl;
        } else if (D == t) {
          if (be < quota) emit(bl + be, i, (int)D);
          ++be;
        }
      }
    }
    run_lt += row_lt;
    run_eq += row_eq;
  }
  __syncthreads();  // warp_tmp and the list are free again
  return tot_lt + min(tot_eq, quota);
}

// Ordered compaction of the block's distances dist_s[0, len) in one pass:
// emits, in ascending index order, every i with D < thr and the first
// `quota` with D == thr, as emit(pos, i, D) with pos the rank among the
// emitted ones; returns their number (compact_block's contract).  Thread t
// counts the tokens below and at thr in its own contiguous run of octets
// (rotated reads, as in compact_block), one block prefix of both counts
// gives its bases, and it emits its tokens in order: no octet list and one
// barrier pair.  dist_s readable 8 entries past len.  All threads call it.
template <typename Emit>
__device__ uint32_t compact_few(const uint16_t* dist_s, int len, int thr, uint32_t quota, uint32_t* warp_tmp,
                                Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int noct = (len + 7) >> 3;
  const uint32_t t = (uint32_t)thr;
  int R = 1;
  while (R * kThreads < noct) R <<= 1;
  const int o0 = tid * R;
  uint32_t fl = 0, lt = 0, eq = 0;
  for (int j = 0; j < R; ++j) {
    const int r = (j + tid) & (R - 1), o = o0 + r;
    if (o >= noct) continue;
    const uint4 v = *reinterpret_cast<const uint4*>(dist_s + 8 * o);
    const uint32_t m = __vminu2(__vminu2(v.x, v.y), __vminu2(v.z, v.w));
    if (min(m & 0xffffu, m >> 16) > t) continue;
    fl |= 1u << r;
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t D = (wd[e >> 1] >> (16 * (e & 1))) & 0xffffu;
      const bool in = 8 * o + e < len;
      lt += (in && D < t) ? 1u : 0u;
      eq += (in && D == t) ? 1u : 0u;
    }
  }
  // block-wide exclusive prefixes of lt and eq
  const uint32_t il = warp_incl_u32(lt), ie = warp_incl_u32(eq);
  __syncthreads();
  if (lane == 31) {
    warp_tmp[warp] = il;
    warp_tmp[kWarps + warp] = ie;
  }
  __syncthreads();
  uint32_t bl = il - lt, be = ie - eq, tot_lt = 0, tot_eq = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = warp_tmp[w], y = warp_tmp[kWarps + w];
    bl += w < warp ? x : 0u;
    be += w < warp ? y : 0u;
    tot_lt += x;
    tot_eq += y;
  }
  while (fl) {
    const int o = o0 + __ffs(fl) - 1;
    fl &= fl - 1;
    const uint4 v = *reinterpret_cast<const uint4*>(dist_s + 8 * o);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t D = (wd[e >> 1] >> (16 * (e & 1))) & 0xffffu;
      const int i = 8 * o + e;
      if (i >= len) continue;
      if (D < t) {
        emit(bl + min(be, quota), i, (int)D);
        ++bl;
      } else if (D == t) {
        if (be < quota) emit(bl + be, i, (int)D);
        ++be;
      }
    }
  }
  __syncthreads();  // warp_tmp is free again
  return tot_lt + min(tot_eq, quota);
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
template <int W>
__device__ __forceinline__ void cp_async_code(uint32_t* dst, const uint32_t* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (W == 4)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(src) : "memory");
}
// Zero-filled instead when !valid (src must still be a valid address).
template <int W>
__device__ __forceinline__ void cp_async_code_zf(uint32_t* dst, const uint32_t* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (W == 4)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(d), "l"(src), "r"(valid ? 8 : 0) : "memory");
}

// Block b serves pair p0 + b / nseg and its candidate range
// [s0, s1) = [(b % nseg) * per_block, ...): no block straddles two pairs.
template <int W, int NP, bool ATTEND, typename T>
__global__ void __launch_bounds__(kThreads, 1) fused_kernel(FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + a.off_hist);
  uint16_t* dist_s = reinterpret_cast<uint16_t*>(smem + a.off_dist);
  int32_t* sel_s = reinterpret_cast<int32_t*>(smem + a.off_sel);
  float* aq_s = reinterpret_cast<float*>(smem + a.off_aq);  // [g][128] attention queries (fp32)
  unsigned char* cscratch = smem + kCompactScratch;  // compaction lists (in the code ring, free by then)
  __nv_bfloat16* qs_s = reinterpret_cast<__nv_bfloat16*>(smem + a.off_qs);  // [kMaxGroup][kQP] bf16 queries
  int* tokw_s = reinterpret_cast<int*>(smem + a.off_tokw);                    // [2][kAW][kWR] rows of the warp steps
  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ __align__(8) uint32_t warp_tmp[3 * kWarps];
  __shared__ int sh[12];
  __shared__ float m_s[kMaxGroup], l_s[kMaxGroup], alpha_s[kMaxGroup];
  __shared__ int tok_s[2 * kRows];

  const int tid = threadIdx.x;
  const int nseg = a.nseg;
  const int p = a.p0 + (int)blockIdx.x / nseg, seg = (int)blockIdx.x % nseg;
  const int64_t kvc = unit_rows(a, p);  // this unit's row key (first cache row when contiguous)
  // Programmatic dependent launch.  The next kernel on this stream may be
  // launched now, so its blocks are ready to take each SM this grid leaves;
  // they wait below until this grid has finished.  Before this block touches
  // global memory, the previous kernel on the stream must have finished with
  // its writes visible (without a programmatic predecessor the wait returns
  // at once).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  HKV_TL(0);
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
  uint32_t* sync = a.sync + kSync * p;

  // ---------------- phase A: small loads first, then the code stream ------
  // Each thread streams its codes (tokens tid, tid + kThreads, ...) through a
  // private ring of kSlots cp.async slots, two codes per commit group.
  // Loads issued before the code stream are ahead of it in the memory queues.
  const int nt = tid < len ? (len - tid + kThreads - 1) / kThreads : 0;
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
  uint32_t* ring = reinterpret_cast<uint32_t*>(smem);
  const uint32_t* pf_ptr = a.ptab != nullptr ? a.k_codes : a.k_codes + (kvc + lo + s0 + tid) * W;  // contiguous only
  constexpr int64_t kStep = (int64_t)kThreads * W;
  auto slot = [&](int k) { return ring + ((size_t)(k % kSlots) * kThreads + tid) * 4; };
  // paged cache: the code of token k of this thread comes through the page
  // table; a page outside the pool zero-fills its slot and marks it in `bad`
  const bool paged = a.ptab != nullptr;
  uint32_t bad = 0, bad_seen = 0;
  // the page ids of the block's scan range go to shared memory (read from
  // the ring's first refill on, after the first block barrier) when they fit
  int* pt_s = reinterpret_cast<int*>(smem + a.off_pt);
  int pj0 = 0;
  bool pt_local = false;
  if (paged && len > 0) {
    const int t0 = lo + s0, t1 = lo + s0 + len - 1;
    pj0 = a.ps_shift >= 0 ? t0 >> a.ps_shift : t0 / a.page_size;
    const int npg = (a.ps_shift >= 0 ? t1 >> a.ps_shift : t1 / a.page_size) - pj0 + 1;
    pt_local = npg <= kPtCap;
    if (pt_local)
      for (int i = tid; i < npg; i += kThreads) pt_s[i] = __ldg(a.ptab + (kvc >> 32) * a.max_pages + pj0 + i);
  }
  auto issue_code = [&](int k) {
    if (!paged) {
      cp_async_code<W>(slot(k), pf_ptr + k * kStep);
      return;
    }
    const int t = lo + s0 + tid + k * kThreads;
    int64_t r;
    if (pt_local && k >= kSlots) {
      int j, sl;
      if (a.ps_shift >= 0) {
        j = t >> a.ps_shift;
        sl = t & (a.page_size - 1);
      } else {
        j = t / a.page_size;
        sl = t - j * a.page_size;
      }
      const int pg = pt_s[j - pj0];
      r = (pg < 0 || (int64_t)pg >= a.num_pages) ? -1
                                                  : ((int64_t)pg * a.Hkv_real + (kvc & 0xffffffffLL)) * a.page_size + sl;
    } else {
      r = cache_row(a, p, kvc, t);
    }
    const uint32_t bit = 1u << (k % kSlots);
    bad = r < 0 ? (bad | bit) : (bad & ~bit);
    cp_async_code_zf<W>(slot(k), a.k_codes + (r < 0 ? 0 : r) * W, r >= 0);
  };
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    if (k < nt) issue_code(k);
    if (k & 1) cp_async_commit();
  }
  if (tid == 0) {
    sh[1] = a.nbins - 1;  // defaults: block hi, speculative bound, count below hi
    sh[3] = a.nbins - 1;
    sh[4] = 0;
    sh[9] = a.nbins - 1;
  }
  const int R_res = sink_n + local_n;
  const int n_res = seg < R_res ? (R_res - seg + nseg - 1) / nseg : 0;
  auto res_row = [&](int i) {  // the block's i-th resident row
    const int v = seg + i * nseg;
    return v < sink_n ? v : local_start + (v - sink_n);
  };
  if (ATTEND && !a.spec && tid < n_res) {
    const int64_t r = cache_row(a, p, kvc, res_row(tid));
    if (r >= 0) prefetch_row_l2<T>(a.K, a.V, r);
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
  HKV_TL(1);
  if constexpr (ATTEND && sizeof(T) == 2) fill_qs(a.g, aq_s, qs_s);  // read only after later barriers
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
      int D0 = token_distance<W, NP>(ck0, planes);
      int D1 = two ? token_distance<W, NP>(ck1, planes) : 0;
      if (paged) {
        // a token on a page outside the pool gets the largest distance
        if ((bad >> (k % kSlots)) & 1u) D0 = a.nbins - 1;
        if (two && ((bad >> ((k + 1) % kSlots)) & 1u)) D1 = a.nbins - 1;
        bad_seen |= bad & ((1u << (k % kSlots)) | (two ? 1u << ((k + 1) % kSlots) : 0u));
      }
      const int j0 = tid + k * kThreads;
      dist_s[j0] = (uint16_t)D0;
      atomicAdd(&hist_s[D0], 1u);
      if (two) {
        dist_s[j0 + kThreads] = (uint16_t)D1;
        atomicAdd(&hist_s[D1], 1u);
      }
      if (k + kSlots < nt) issue_code(k + kSlots);
      if (k + 1 + kSlots < nt) issue_code(k + 1 + kSlots);
      cp_async_commit();
    }
    cp_async_wait<0>();
    if (bad_seen) report(a.status, HKV_ERR_DEVICE_RANGE);
  }
  __syncthreads();
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
  HKV_TL(2);

  // ---------------- publication -----------------------------------------------
  // The segment adds its histogram counts up to hi (its own k-th smallest D,
  // or all bins if it holds fewer than k_eff tokens) into the pair's global
  // histogram, and stores its cumulative counts over [0, hi].  The pair's
  // threshold T is at most min over segments of hi (that segment alone has
  // k_eff tokens at or below its hi), so the global histogram is complete on
  // [0, T] and every segment's cumulative counts are known at T - 1 and T.
  const uint32_t k_eff = (uint32_t)k_eff_p;
  const int spec_cap = kRows - n_res;  // speculative rows that fit beside the resident ones in one tile
  int hi, tb;
  // this block's proportional share of the selection (for the threshold estimate)
  const uint32_t share = C > 0 ? (uint32_t)max(1ll, ((long long)k_eff * len + C - 1) / C) : 1u;
  {
    uint32_t cnt[4], cum[4];
    const uint4 hv = 4 * tid < a.nbins_pad ? *reinterpret_cast<const uint4*>(hist_s + 4 * tid) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t total = hist_cum4(hv, cnt, cum, warp_tmp);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int v = 4 * tid + e;
      if (v < a.nbins) {
        if (k_eff > 0u && cum[e] >= k_eff && cum[e] - cnt[e] < k_eff) {
          sh[1] = v;
          sh[4] = (int)(cum[e] - cnt[e]);
        }
        // estimate of the pair's threshold: where this block holds its share of k_eff
        if (cum[e] >= share && cum[e] - cnt[e] < share) sh[9] = v;
        // speculative bound: the largest bin whose cumulative count fits spec_cap
        if (cum[e] > (uint32_t)max(spec_cap, 0) && cum[e] - cnt[e] <= (uint32_t)max(spec_cap, 0)) sh[3] = v - 1;
      }
    }
    __syncthreads();
    // k_eff == 0 (a ragged sequence without candidates): nothing to publish
    hi = k_eff == 0u ? -1 : total >= k_eff ? sh[1] : a.nbins - 1;
    tb = spec_cap > 0 ? sh[3] : -1;
    if (nseg > 1) {
      uint32_t* cum_out = a.cum + ((int64_t)p * nseg + seg) * a.nbins_pad;
      uint32_t* gh = a.gh + (int64_t)p * a.nbins_pad;
      if (4 * tid + 3 <= hi) {
        *reinterpret_cast<uint4*>(cum_out + 4 * tid) = make_uint4(cum[0], cum[1], cum[2], cum[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * tid + e <= hi) cum_out[4 * tid + e] = cum[e];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (4 * tid + e <= hi && cnt[e] != 0u) red_add_gpu(&gh[4 * tid + e], cnt[e]);
      __syncthreads();
      if (tid == 0 && !(a.skip_arrive && blockIdx.x == 0)) red_release_add(&sync[0], 1u);
    }
    // (one block per pair: its own k-th smallest distance is the threshold,
    // nothing is exchanged)
    HKV_TL(3);
  }

  // ---------------- speculative tile -----------------------------------------
  // While the other blocks publish, the block gathers the K/V rows of its
  // tokens with D <= tb (tb: the largest bin whose cumulative count fits
  // beside its resident rows in one tile) and of its resident rows.  When the
  // pair's threshold turns out to be <= tb, every selected token of the block
  // is in this tile and the attention needs no further gather.
  int n_spec = 0;
  auto spec_row = [&](int i) -> int { return i < n_spec ? sel_s[i] : res_row(i - n_spec); };
  if constexpr (ATTEND && sizeof(T) == 2) {
    if (a.spec) {
      n_spec = (int)compact_few(dist_s, len, tb + 1, 0u, warp_tmp, [&](uint32_t pos, int i, int) {
        if (pos < (uint32_t)kRows) sel_s[pos] = lo + s0 + i;
      });
      n_spec = min(n_spec, max(spec_cap, 0));
      __syncthreads();
      HKV_TL(11);
      if ((tid >> 5) < kAW && (tid >> 5) * kWR < n_spec + n_res)  // slot 0 of warps 0-3
        warp_issue(a, p, kvc, n_spec + n_res, spec_row, tid >> 5, smem + (size_t)(tid >> 5) * kSlotBytes,
                   tokw_s + (tid >> 5) * kWR);
      HKV_TL(12);
    }
  }

  // ---------------- phase B: threshold and ordered compaction ---------------
  uint32_t n_sel = 0, sel_base = 0;
  bool spec_ok = false;
  if (nseg > 1) {
    if (tid == 0) sh[2] = wait_count(&sync[0], (uint32_t)nseg, a.wait_ns) ? 1 : 0;
    __syncthreads();
  }
  HKV_TL(4);
  const bool arrived = nseg == 1 || sh[2] != 0;
  if (arrived) {
    int thr = max(hi, 0);
    uint32_t below = (uint32_t)sh[4];
    // lower segments' cumulative counts over a window of 8 bins around this
    // block's estimate of T, loaded in the same round as the pair histogram
    // (pairs of at most kThreads / 8 blocks: one load per thread)
    const int w0 = max(0, sh[9] - 5);
    const bool win = seg <= kThreads / 8;
    const int wss = tid >> 3, wj = tid & 7;
    const uint32_t wv = win && wss < seg && w0 + wj < a.nbins
                            ? __ldcg(a.cum + ((int64_t)p * nseg + wss) * a.nbins_pad + w0 + wj)
                            : 0u;
    if (nseg > 1) {
      // the pair's histogram: four bins per thread, one load round
      uint32_t cnt[4], cum[4];
      const uint32_t* gh = a.gh + (int64_t)p * a.nbins_pad;
      const uint4 gv = 4 * tid < a.nbins_pad ? __ldcg(reinterpret_cast<const uint4*>(gh) + tid) : make_uint4(0u, 0u, 0u, 0u);
      if (tid == 0) {
        sh[5] = a.nbins - 1;
        sh[6] = 0;
      }
      hist_cum4(gv, cnt, cum, warp_tmp);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int v = 4 * tid + e;
        if (v < a.nbins && cum[e] >= k_eff && cum[e] - cnt[e] < k_eff) {
          sh[5] = v;
          sh[6] = (int)(cum[e] - cnt[e]);
        }
      }
      __syncthreads();
      thr = sh[5];
      below = (uint32_t)sh[6];
    }
    // tokens of the lower segments below and at the threshold (from the
    // window when it holds T - 1 and T; values past a segment's hi are stale
    // but never used: T <= every segment's hi)
    uint32_t seg_lt = 0, seg_le = 0;
    if (win && thr >= w0 && thr <= w0 + 7 && (thr == 0 || thr - 1 >= w0)) {
      if (wss < seg) {
        if (wj == thr - w0) seg_le += wv;
        if (wj == thr - 1 - w0) seg_lt += wv;
      }
    } else {
      for (int ss = tid; ss < seg; ss += kThreads) {
        const uint32_t* c = a.cum + ((int64_t)p * nseg + ss) * a.nbins_pad;
        seg_lt += thr > 0 ? __ldcg(c + thr - 1) : 0u;
        seg_le += __ldcg(c + thr);
      }
    }
    block_sum2(seg_lt, seg_le, warp_tmp);
    const uint32_t lower_lt = seg_lt, lower_eq = seg_le - seg_lt;
    const uint32_t ties_needed = k_eff - below;
    const uint32_t quota = ties_needed > lower_eq ? ties_needed - lower_eq : 0u;
    sel_base = lower_lt + min(lower_eq, ties_needed);
    HKV_TL(5);
    int32_t* idx_out = a.idx + (int64_t)p * a.top_k + sel_base;
    int32_t* dist_out = a.dist ? a.dist + (int64_t)p * a.top_k + sel_base : nullptr;
    if (ATTEND && a.spec && thr <= tb) {
      // every selected token of the block has D <= thr <= tb, so it is in the
      // speculative list (ascending); keep D < thr, and ties at thr in
      // order up to the quota; mask the others out of the tile
      spec_ok = true;
      if (tid < 32) {
        const int lane = tid;
        uint32_t run = 0, run_eq = 0;
        for (int i0 = 0; i0 < n_spec; i0 += 32) {
          const int i = i0 + lane;
          const bool valid = i < n_spec;
          const int tok = valid ? sel_s[i] : 0;
          const uint32_t D = valid ? dist_s[tok - lo - s0] : 0xffffu;
          const bool is_eq = valid && D == (uint32_t)thr;
          const uint32_t eq_rank = run_eq + __popc(__ballot_sync(0xffffffffu, is_eq) & lanemask_lt());
          const bool take = valid && (D < (uint32_t)thr || (is_eq && eq_rank < quota));
          const uint32_t tm = __ballot_sync(0xffffffffu, take);
          const uint32_t pos = run + __popc(tm & lanemask_lt());
          if (take) {
            if (sel_base + pos < k_eff) {
              idx_out[pos] = tok;
              if (dist_out) dist_out[pos] = (int32_t)D;
            } else {
              report(a.status, HKV_ERR_DEVICE_RANGE);  // unreachable when the counts agree
            }
          }
          if (valid && !take) tokw_s[i] = -1;
          run += __popc(tm);
          run_eq += __popc(__ballot_sync(0xffffffffu, is_eq));
        }
        if (lane == 0) sh[7] = (int)run;
      }
      __syncthreads();
      n_sel = (uint32_t)sh[7];
    } else {
      if constexpr (ATTEND && sizeof(T) == 2) {
        if (a.spec) cp_async_wait<0>();  // the speculative tile is not used
      }
      auto emit = [&](uint32_t pos, int i, int D) {
        const int tok = lo + s0 + i;
        if (sel_base + pos < k_eff) {
          idx_out[pos] = tok;
          if (dist_out) dist_out[pos] = D;
          if constexpr (ATTEND) {
            if (pos < (uint32_t)a.sel_cap) sel_s[pos] = tok;
          }
        } else {
          report(a.status, HKV_ERR_DEVICE_RANGE);  // unreachable when the counts agree
        }
      };
      // short runs per thread (at most two octets): one pass; longer runs
      // balance better through the octet list
      n_sel = len <= 16 * kThreads ? compact_few(dist_s, len, thr, quota, warp_tmp, emit)
                                   : compact_block(dist_s, len, thr, quota, warp_tmp, cscratch, emit);
      if (sel_base + n_sel > k_eff) n_sel = k_eff > sel_base ? k_eff - sel_base : 0u;
    }
  } else {
    if (tid == 0) report(a.status, HKV_ERR_TIMEOUT);
    if constexpr (ATTEND && sizeof(T) == 2) {
      if (a.spec) cp_async_wait<0>();  // no copy may land after the block exits
    }
  }
  __syncthreads();
  HKV_TL(6);

  if constexpr (ATTEND) {
    if (arrived) {
      // ---------------- attention over selected + resident rows, partial -----
      const int ns = (int)n_sel;
      const int32_t* sel_g = a.idx + (int64_t)p * a.top_k + sel_base;
      auto row_at = [&](int i) -> int {
        if (i < ns) return i < a.sel_cap ? sel_s[i] : sel_g[i];
        return res_row(i - ns);
      };
      float* part_s = reinterpret_cast<float*>(smem + a.off_part);
      float* dst = nseg == 1 ? part_s : a.part + ((int64_t)p * nseg + seg) * a.g * kPart;
      if constexpr (sizeof(T) == 2) {
        if (spec_ok) {
          attn_warps(a, p, kvc, n_spec + n_res, spec_row, smem, tokw_s, qs_s, dst, (n_spec + n_res + kWR - 1) / kWR);
        } else {
          attn_warps(a, p, kvc, ns + n_res, row_at, smem, tokw_s, qs_s, dst, 0);
        }
      } else {
        float* attn = reinterpret_cast<float*>(smem);
        const AttnSmem sm{aq_s, attn, attn + kRows * kKP, attn + kRows * kKP + kRows * kHeadDim, tok_s, m_s, l_s, alpha_s};
        float acc[kOut];
        attn_begin(a.g, sm, acc);
        attn_rows<T>(a, p, kvc, ns + n_res, row_at, sm, acc);
        attn_end(a.g, sm, acc, dst);
      }
      __syncthreads();
      HKV_TL(7);
      bool last = nseg == 1;
      if (nseg == 1) {
        finish_single(a, p, part_s);
      } else {
        // the last blocks of the pair to finish merge a run of its output
        // columns each (merge_split, merge_cols); the
        // last of them to finish returns the pair's counters and histogram to
        // zero (every block is past its last use of them)
        if (tid == 0) sh[8] = (int)atom_acq_rel_add(&sync[2], 1u);
        __syncthreads();
        const MergeSplit ms = merge_split(a.g, nseg);
        const int nm = ms.nm;
        const int mi = sh[8] - (nseg - nm);
        if (mi >= 0) {
          if (tid == 0) sh[7] = wait_count(&sync[2], (uint32_t)nseg, a.wait_ns) ? 1 : 0;
          __syncthreads();
          HKV_TL(8);
          if (sh[7]) {
            merge_share(a.part, a.out, a.lse, a.Hq, a.Hkv, a.g, p, nseg, mi, ms, reinterpret_cast<float*>(smem));
          } else if (tid == 0) {
            report(a.status, HKV_ERR_TIMEOUT);
          }
          HKV_TL(9);
          if (tid == 0) sh[7] = atomicAdd(&sync[3], 1u) == (uint32_t)(nm - 1) ? 1 : 0;
          __syncthreads();
          last = sh[7] != 0;
        }
      }
      if (last) {
        for (int i = k_eff_p + tid; i < a.top_k; i += kThreads) a.idx[(int64_t)p * a.top_k + i] = -1;
        for (int v = tid; v < a.nbins_pad; v += kThreads) a.gh[(int64_t)p * a.nbins_pad + v] = 0u;
        if (tid == 0) {
          sync[0] = 0u;
          sync[2] = 0u;
          sync[3] = 0u;
        }
      }
      HKV_TL(10);
      return;
    }
  }

  // ---------------- departure; the last block out resets the counters -------
  // (retrieval only, or after a timeout)
  __syncthreads();
  if (tid == 0) sh[2] = atom_acq_rel_add(&sync[1], 1u) == (uint32_t)(nseg - 1);
  __syncthreads();
  if (sh[2]) {
    for (int i = k_eff_p + tid; i < a.top_k; i += kThreads) {
      a.idx[(int64_t)p * a.top_k + i] = -1;
      if (a.dist) a.dist[(int64_t)p * a.top_k + i] = -1;
    }
    for (int v = tid; v < a.nbins_pad; v += kThreads) a.gh[(int64_t)p * a.nbins_pad + v] = 0u;
    if (tid == 0) {
      sync[0] = 0u;
      sync[1] = 0u;
    }
  }
  HKV_TL(10);
}

// ---------------- standalone sparse attention (bf16) --------------------------
// hkv_sparse_attend and hkv_sparse_attend_paged for bf16 caches on the fused
// kernel's attention stage (Spotlight Attention "Approach": exact attention
// over the retrieved tokens with the sink and local rows; RetrievalAttention
// "Summary", "Approach": partial results merged by log-sum-exp rescaling).
// Block x serves pair p = p0 + x / nseg and rows [seg * per_block, ...) of
// the pair's row list [sink | idx slots | local]; eight warps take 16-row
// steps with two cp.async slots each (attn_warps).  One segment per pair
// writes out / lse itself; with several (a cooperative launch) the last
// blocks of the pair merge a run of its output columns each, as in the
// fused kernel.
constexpr int kSaTok = 4096;  // row tokens kept in shared memory per block

struct SaLayout {
  static constexpr size_t qs = kAttnWarpBytes;                                   // bf16 [16][kQP]
  static constexpr size_t tokw = qs + (size_t)kMaxGroup * kQP * 2;              // int [2][kAW][kWR]
  static constexpr size_t tok = tokw + (size_t)2 * kAW * kWR * 4;               // int [kSaTok]
  static constexpr size_t part = tok + (size_t)kSaTok * 4;                      // float [g][kPart]
  static constexpr size_t total = part + (size_t)kMaxGroup * kPart * 4;
};

__global__ void __launch_bounds__(kThreads, 1) sattend_kernel(FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // programmatic dependent launch, as in fused_kernel: the next kernel may
  // launch now; this block reads global memory only after the previous
  // kernel on the stream has finished
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  __nv_bfloat16* qs_s = reinterpret_cast<__nv_bfloat16*>(smem + SaLayout::qs);
  int* tokw_s = reinterpret_cast<int*>(smem + SaLayout::tokw);
  int* tok_s = reinterpret_cast<int*>(smem + SaLayout::tok);
  float* part_s = reinterpret_cast<float*>(smem + SaLayout::part);
  __shared__ int sh[2];
  const int tid = threadIdx.x, g = a.g;
  const int p = a.p0 + (int)(blockIdx.x / a.nseg), seg = (int)(blockIdx.x % a.nseg);
  const int nseg = a.nseg;
  const int64_t Rv = (int64_t)a.sink_n + a.top_k + a.local_n;
  const int64_t v0 = (int64_t)seg * a.per_block;
  const int nrows = (int)max((int64_t)0, min((int64_t)a.per_block, Rv - v0));
  // token of row v of the pair's list (-1: an empty idx slot or a token past N)
  auto token_of = [&](int64_t v) -> int {
    if (v < a.sink_n) return (int)v;
    if (v < (int64_t)a.sink_n + a.top_k) {
      const int t = __ldg(a.idx + (int64_t)p * a.top_k + (v - a.sink_n));
      if (t >= a.C) {
        report(a.status, HKV_ERR_DEVICE_RANGE);
        return -1;
      }
      return t < 0 ? -1 : t;
    }
    return a.local_start + (int)(v - a.sink_n - a.top_k);
  };
  for (int i = tid; i < min(nrows, kSaTok); i += kThreads) tok_s[i] = token_of(v0 + i);
  const int b = p / a.Hkv, kvh = p % a.Hkv;
  const __nv_bfloat16* q0 = tptr<__nv_bfloat16>(a.q) + ((int64_t)b * a.Hq + (int64_t)kvh * g) * kHeadDim;
  for (int i = tid; i < kMaxGroup * kHeadDim; i += kThreads) {
    const int h = i / kHeadDim, k = i % kHeadDim;
    qs_s[h * kQP + k] = h < g ? q0[(int64_t)h * kHeadDim + k] : __float2bfloat16_rn(0.f);
  }
  const int64_t kvc = unit_rows(a, p);
  float* dst = nseg == 1 ? part_s : a.part + ((int64_t)p * nseg + seg) * g * kPart;
  // (attn_warps starts with a block barrier: tok_s and qs_s are complete)
  attn_warps(a, p, kvc, nrows, [&](int i) -> int { return i < kSaTok ? tok_s[i] : token_of(v0 + i); }, smem,
             tokw_s, qs_s, dst, 0);
  if (nseg == 1) {
    finish_single(a, p, part_s);
    return;
  }
  uint32_t* sync = a.sync + kSync * p;
  if (tid == 0) sh[0] = (int)atom_acq_rel_add(&sync[2], 1u);
  __syncthreads();
  const MergeSplit ms = merge_split(g, nseg);
  const int nm = ms.nm;
  const int mi = sh[0] - (nseg - nm);
  if (mi < 0) return;
  if (tid == 0) sh[1] = wait_count(&sync[2], (uint32_t)nseg, a.wait_ns) ? 1 : 0;
  __syncthreads();
  if (sh[1]) {
    merge_share(a.part, a.out, a.lse, a.Hq, a.Hkv, g, p, nseg, mi, ms, reinterpret_cast<float*>(smem));
  } else if (tid == 0) {
    report(a.status, HKV_ERR_TIMEOUT);
  }
  if (tid == 0 && atomicAdd(&sync[3], 1u) == (uint32_t)(nm - 1)) {
    sync[2] = 0u;  // every block of the pair is past its last use of the counters
    sync[3] = 0u;
  }
}

// ---------------- norm-weighted decode step (sign-VQ, bf16) ------------------
// One block per (batch, KV head) pair, windows of at most 65536 candidates:
// the group's sign query codes by ballots, the norm-weighted top-k of
// normw_select.cuh (Self-Indexing KVCache, "Abstract"), then the attention
// over [sink | selected | local] on the tensor cores (attn_warps) and out /
// lse from the block's own partial.  The selection's shared memory is reused
// by the attention.
struct NwDecodeArgs {
  const uint16_t* norms;  // [B, Hkv, cap] fp16
  int gb;                 // g * code bits
  int vec_norms;          // norm rows start on 16-byte boundaries
  float* score;           // nullable [B, Hkv, top_k]
  uint32_t* q_codes_out;  // nullable [B, Hq, W]
};

struct NdLayout {
  static constexpr size_t qs = kAttnWarpBytes;                       // bf16 [16][kQP]
  static constexpr size_t tokw = qs + (size_t)kMaxGroup * kQP * 2;  // int [2][kAW][kWR]
  static constexpr size_t part = tokw + (size_t)2 * kAW * kWR * 4;  // float [g][kPart]
  static constexpr size_t attn = part + (size_t)kMaxGroup * kPart * 4;
};

template <int W, int NP>
__global__ void __launch_bounds__(kThreads, 1) normw_decode_kernel(FusedArgs a, NwDecodeArgs n) {
  extern __shared__ __align__(128) unsigned char smem[];
  // programmatic dependent launch, as in fused_kernel: the next kernel may
  // launch now; this block reads global memory only after the previous
  // kernel on the stream has finished
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  __shared__ uint32_t qc_s[kMaxGroup * W];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t found[3];
  __shared__ uint32_t cnt_s[2 * kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = a.g;
  const int p = blockIdx.x, b = p / a.Hkv, kvh = p % a.Hkv;
  const int k_eff = a.k_eff;
  int32_t* idx = a.idx + (int64_t)p * a.top_k;
  float* score = n.score != nullptr ? n.score + (int64_t)p * a.top_k : nullptr;
  for (int i = k_eff + tid; i < a.top_k; i += kThreads) {
    idx[i] = -1;
    if (score != nullptr) score[i] = -INFINITY;
  }
  const int64_t qrow0 = (int64_t)b * a.Hq + (int64_t)kvh * g;
  const __nv_bfloat16* q0 = tptr<__nv_bfloat16>(a.q) + qrow0 * kHeadDim;
  for (int r = warp; r < g; r += kWarps) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const uint32_t word = __ballot_sync(0xffffffffu, __bfloat162float(q0[(int64_t)r * kHeadDim + lane + 32 * w]) > 0.f);
      if (lane == 0) qc_s[r * W + w] = word;
    }
  }
  __syncthreads();
  if (n.q_codes_out != nullptr)
    for (int i = tid; i < g * W; i += kThreads) n.q_codes_out[qrow0 * W + i] = qc_s[i];
  const int64_t kvc = unit_rows(a, p);
  if (k_eff > 0)
    nw::block_select<W, NP>(a.k_codes + (kvc + a.lo) * W, n.norms + kvc + a.lo, n.vec_norms != 0, qc_s, g, n.gb,
                            (int)a.lo, a.C, k_eff, smem, wsum, found, cnt_s, idx, score);
  __syncthreads();  // idx is complete; the selection's shared memory is free
  __nv_bfloat16* qs_s = reinterpret_cast<__nv_bfloat16*>(smem + NdLayout::qs);
  int* tokw_s = reinterpret_cast<int*>(smem + NdLayout::tokw);
  float* part_s = reinterpret_cast<float*>(smem + NdLayout::part);
  for (int i = tid; i < kMaxGroup * kHeadDim; i += kThreads) {
    const int h = i / kHeadDim, k = i % kHeadDim;
    qs_s[h * kQP + k] = h < g ? q0[(int64_t)h * kHeadDim + k] : __float2bfloat16_rn(0.f);
  }
  const int nrows = a.sink_n + k_eff + a.local_n;
  const int32_t* sel = idx;  // written by this block (plain loads, not the read-only path)
  attn_warps(a, p, kvc, nrows,
             [&](int i) -> int {
               if (i < a.sink_n) return i;
               if (i < a.sink_n + k_eff) return sel[i - a.sink_n];
               return a.local_start + (i - a.sink_n - k_eff);
             },
             smem, tokw_s, qs_s, part_s, 0);
  finish_single(a, p, part_s);
}

struct SaPlan {
  int nseg = 1, per_block = 0, pairs_per_launch = 1;
  bool cooperative = false;
  size_t ws_part = 0, ws_sync = 0, ws_total = 0;
};

SaPlan sattend_plan(const AttendShape& s) {
  SaPlan pl;
  const Window w = window(s.N, s.n_sink, s.n_local);
  const int g = s.Hq / s.Hkv, P = s.B * s.Hkv;
  const int64_t Rv = std::max<int64_t>(1, w.sink_end + s.top_k + (s.N - w.local_start));
  const int G = sm_count();
  // at least one 16-row step per warp and block; one wave of blocks when a
  // pair is split (its blocks wait for each other)
  int64_t nseg = 1;
  if (P > 0 && P < G) nseg = std::max<int64_t>(1, std::min<int64_t>(G / P, ceil_div(Rv, (int64_t)kAW * kWR)));
  nseg = std::min<int64_t>(nseg, kMaxSegsPerPair);
  pl.per_block = (int)ceil_div(Rv, nseg);
  pl.nseg = (int)ceil_div(Rv, pl.per_block);
  pl.cooperative = pl.nseg > 1;
  pl.pairs_per_launch = pl.cooperative ? std::max(1, G / pl.nseg) : std::max(P, 1);
  pl.ws_part = pl.nseg > 1 ? align_up(sizeof(float) * (size_t)P * pl.nseg * g * kPart, 256) : 0;
  pl.ws_sync = align_up(sizeof(uint32_t) * kSync * (size_t)std::max(P, 1), 256);
  pl.ws_total = pl.ws_part + pl.ws_sync;
  return pl;
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
  int nseg, per_block, pairs_per_launch, sel_cap;
  bool cooperative;
  uint32_t off_q, off_aq, off_sel, off_hist, off_dist, off_part, off_qs, off_tokw, off_pt;
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
  // Shared memory: a region written during the scan and the selection and
  // dead afterwards (code ring at 0, query-encode staging, histogram,
  // distances, chunk minima), which the attention then reuses from offset 0;
  // then the arrays that live to the end (attention queries, selected rows,
  // the single-block partial, bf16 queries, warp-step rows).
  const size_t attn = attend ? std::max(sizeof(float) * (kRows * kKP + kRows * kHeadDim + kMaxGroup * kRows),
                                        kAttnWarpBytes)
                              : 0;
  const size_t budget = (size_t)max_smem_optin() - kStaticSmem;
  bool fits = false;
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
    pl.sel_cap = attend ? (int)align_up((size_t)std::max(kRows, std::min(kSelCap, pl.k_eff)), 64) : 0;
    size_t qst = 0;
    if (q_elt == 2) qst = align_up(sizeof(uint16_t) * (kQRows + bits) * (kHeadDim + 8) + kQRows * bits / 8, 16);
    if (q_elt == 4) qst = align_up(sizeof(float) * (kQRows * kHeadDim + bits * (kHeadDim + 1)), 16);
    size_t off = (size_t)kSlots * kThreads * 16;  // code ring
    pl.off_q = (uint32_t)off;
    off += qst;
    pl.off_hist = (uint32_t)off;
    off += sizeof(uint32_t) * 2 * (size_t)pl.nbins_pad;
    pl.off_dist = (uint32_t)off;
    off += align_up(sizeof(uint16_t) * ((size_t)pl.per_block + 16), 16);  // vector reads run past the end
    off = std::max(off, attn);
    pl.off_aq = (uint32_t)off;
    if (attend) off += align_up(sizeof(float) * pl.g * kHeadDim, 16);
    pl.off_sel = (uint32_t)off;
    off += align_up(sizeof(int32_t) * (size_t)pl.sel_cap, 16);
    pl.off_part = (uint32_t)off;
    if (attend && pl.nseg == 1) off += sizeof(float) * pl.g * kPart;
    pl.off_qs = (uint32_t)off;
    if (attend) off += align_up(sizeof(uint16_t) * kMaxGroup * kQP, 16);
    pl.off_tokw = (uint32_t)off;
    if (attend) off += sizeof(int) * 2 * kAW * kWR;
    pl.off_pt = (uint32_t)off;
    if (s.pm != nullptr) off += sizeof(int) * kPtCap;
    pl.smem = align_up(off, 16);
    fits = pl.smem <= budget;
    if (fits) break;
  }
  if (!fits) return fail(HKV_ERR_UNSUPPORTED, "the scan kernel's shared memory does not fit for this shape");
  pl.ws_sync = align_up(sizeof(uint32_t) * kSync * P, 256);
  pl.ws_gh = align_up(sizeof(uint32_t) * (size_t)P * pl.nbins_pad, 256);
  pl.ws_cum = align_up(sizeof(uint32_t) * (size_t)P * pl.nseg * pl.nbins_pad, 256);
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
  a.off_part = pl.off_part;
  a.off_qs = pl.off_qs;
  a.off_tokw = pl.off_tokw;
  a.off_pt = pl.off_pt;
  a.sel_cap = pl.sel_cap;
  {
    // speculative tile: when a block's expected share of the selection, with
    // a two-fold margin, fits one tile beside its resident rows
    const int64_t res = (int64_t)w.sink_end + (s.N - w.local_start);
    const int64_t res_blk = ceil_div(res, pl.nseg);
    a.spec = attend && dtype == HKV_BF16 && pl.nseg > 1 && 2 * ceil_div(pl.k_eff, pl.nseg) + res_blk <= kRows ? 1 : 0;
  }
  a.sync = reinterpret_cast<uint32_t*>(base);
  a.gh = reinterpret_cast<uint32_t*>(base + pl.ws_sync);
  a.cum = reinterpret_cast<uint32_t*>(base + pl.ws_sync + pl.ws_gh);
  a.part = reinterpret_cast<float*>(base + pl.ws_sync + pl.ws_gh + pl.ws_cum);
  a.status = status;
  a.wait_ns = wait_limit_ns();
  if (s.pm != nullptr) {
    a.ptab = s.pm->table;
    a.max_pages = s.pm->max_pages;
    a.num_pages = s.pm->num_pages;
    a.page_size = s.pm->page_size;
    a.ps_shift = -1;
    if ((a.page_size & (a.page_size - 1)) == 0) {
      a.ps_shift = 0;
      while ((1 << a.ps_shift) < a.page_size) ++a.ps_shift;
    }
    a.next_codes = nullptr;  // the hint is for contiguous caches
  }
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

int launch_normw_decode(const RetrieveShape& s, const void* q, const uint32_t* k_codes, const uint16_t* norms,
                        const void* K, const void* V, float scale, uint32_t* q_codes, int32_t* idx, float* score,
                        float* out, float* lse, int32_t* status, cudaStream_t st) {
  const int P = s.B * s.Hkv;
  if (P == 0 || s.top_k == 0) return HKV_OK;
  const Window w = window(s.N, s.n_sink, s.n_local);
  if (w.C > nw::kMaxTokens)
    return fail(HKV_ERR_UNSUPPORTED, "%lld candidates per KV head for the one-launch step", (long long)w.C);
  const int g = s.Hq / s.Hkv;
  int np = 0;
  while ((1 << np) <= g) ++np;
  FusedArgs a = {};
  a.k_codes = k_codes;
  a.idx = idx;
  a.q = q;
  a.K = K;
  a.V = V;
  a.out = out;
  a.lse = lse;
  a.scale = scale;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = g;
  a.cap = s.cap;
  a.lo = w.sink_end;
  a.C = (int)w.C;
  a.k_eff = (int)std::min<int64_t>(s.top_k, w.C);
  a.top_k = s.top_k;
  a.sink_n = (int)w.sink_end;
  a.local_start = (int)w.local_start;
  a.local_n = (int)(s.N - w.local_start);
  a.Hkv_real = s.Hkv;
  a.unit_div = 1;
  a.status = status;
  a.ps_shift = -1;
  NwDecodeArgs n;
  n.norms = norms;
  n.gb = g * s.words * 32;
  n.vec_norms = (reinterpret_cast<uintptr_t>(norms) % 16 == 0 && s.cap % 8 == 0 && w.sink_end % 8 == 0) ? 1 : 0;
  n.score = score;
  n.q_codes_out = q_codes;
  using Fn = void (*)(FusedArgs, NwDecodeArgs);
  Fn fn = nullptr;
#define HKV_ND(WV, NPV) \
  if (s.words == WV && np == NPV) fn = normw_decode_kernel<WV, NPV>;
  HKV_ND(2, 1) HKV_ND(2, 2) HKV_ND(2, 3) HKV_ND(2, 4) HKV_ND(2, 5)
  HKV_ND(4, 1) HKV_ND(4, 2) HKV_ND(4, 3) HKV_ND(4, 4) HKV_ND(4, 5)
#undef HKV_ND
  if (fn == nullptr) return fail(HKV_ERR_UNSUPPORTED, "no kernel for %d-bit codes and group %d", s.words * 32, g);
  const int64_t range = ceil_div(std::max<int64_t>(w.C, 1), (int64_t)nw::kWarps * nw::kChunk) * nw::kChunk;
  const size_t sel_smem = nw::kRegionBytes + (size_t)nw::kBins * 4 + (size_t)nw::kWarps * range * 2;
  const size_t smem = std::max(sel_smem, NdLayout::attn);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "norm-weighted decode shared memory");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, fn, a, n), "norm-weighted decode launch");
}

size_t sattend_ws_bytes(const AttendShape& s) { return sattend_plan(s).ws_total; }

int launch_sattend(const AttendShape& s, const void* q, const void* K, const void* V, const int32_t* idx, float scale,
                   float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status, cudaStream_t st,
                   const PageMap* pm) {
  const int P = s.B * s.Hkv;
  if (P == 0) return HKV_OK;
  const SaPlan pl = sattend_plan(s);
  if (ws == nullptr || ws_bytes < pl.ws_total)
    return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, pl.ws_total);
  const Window w = window(s.N, s.n_sink, s.n_local);
  FusedArgs a = {};
  a.q = q;
  a.K = K;
  a.V = V;
  a.idx = const_cast<int32_t*>(idx);
  a.out = out;
  a.lse = lse;
  a.scale = scale;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.g = s.Hq / s.Hkv;
  a.cap = s.cap;
  a.C = (int)std::min<int64_t>(s.N, INT32_MAX);  // tokens: idx entries at or past it are reported
  a.top_k = s.top_k;
  a.sink_n = (int)w.sink_end;
  a.local_start = (int)w.local_start;
  a.local_n = (int)(s.N - w.local_start);
  a.nseg = pl.nseg;
  a.per_block = pl.per_block;
  a.Hkv_real = s.Hkv;
  a.unit_div = 1;
  unsigned char* base = static_cast<unsigned char*>(ws);
  a.part = reinterpret_cast<float*>(base);
  a.sync = reinterpret_cast<uint32_t*>(base + pl.ws_part);
  a.status = status;
  a.wait_ns = wait_limit_ns();
  a.ps_shift = -1;
  if (pm != nullptr) {
    a.ptab = pm->table;
    a.max_pages = pm->max_pages;
    a.num_pages = pm->num_pages;
    a.page_size = pm->page_size;
    if ((a.page_size & (a.page_size - 1)) == 0) {
      a.ps_shift = 0;
      while ((1 << a.ps_shift) < a.page_size) ++a.ps_shift;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(sattend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SaLayout::total);
  if (e != cudaSuccess) return cuda_check(e, "sparse attention shared memory");
  for (int p0 = 0; p0 < P; p0 += pl.pairs_per_launch) {
    a.p0 = p0;
    const int np = P - p0 < pl.pairs_per_launch ? P - p0 : pl.pairs_per_launch;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(np * pl.nseg));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SaLayout::total;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pl.cooperative ? 2 : 1;
    const int rc = cuda_check(cudaLaunchKernelEx(&cfg, sattend_kernel, a), "sparse attention launch");
    if (rc != HKV_OK) return rc;
  }
  return HKV_OK;
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

#ifdef HKV_TIMELINE
extern "C" int hkv_debug_timeline(unsigned long long* dst, int n) {
  const size_t cap = sizeof(hkv::g_hkv_tl) / sizeof(unsigned long long);
  return cudaMemcpyFromSymbol(dst, hkv::g_hkv_tl, sizeof(unsigned long long) * ((size_t)n < cap ? (size_t)n : cap)) ==
                 cudaSuccess
             ? 0
             : -4;
}
#endif
