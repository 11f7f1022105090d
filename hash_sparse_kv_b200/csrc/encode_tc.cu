// LSH key encoder on the tensor cores (HashEvict, "Abstract": the code of a
// key is the sign pattern of its Gaussian random projection R k).
//
// Y = X R^T is a dense [rows x 128] x [128 x bits] contraction, so it runs as
// tcgen05 MMAs (M = 128 rows, N = bits, K = 128 in eight 16-wide steps) with
// bf16 operands and an fp32 accumulator in tensor memory.  bf16 x bf16
// products are exact in fp32; only the fp32 summation order differs from a
// plain dot product, far below the 1e-3 input margin of the sign test.
//
// Persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: R once, then 128-row key tiles into a 4-stage ring
//   warp 1      allocates TMEM; one thread issues the MMAs of each tile into one
//               of two accumulators and commits them to the tile's barriers
//   warps 2..5  epilogue: TMEM -> registers (one row per thread), sign bits
//               packed into uint32 words, one vector store per row
// The key stream is the only large traffic (256 bytes in, 16 bytes out per
// 128-bit code), so the kernel is bound by HBM reads.
#include <cstdio>
#include <mutex>

#include "internal.h"
#include "tc.cuh"

namespace hkv {
namespace {

constexpr int kTcThreads = 192;
constexpr int kTcStages = 4;
constexpr int kTileRows = 128;                      // MMA M
constexpr uint32_t kBoxBytes = kTileRows * 128;     // 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2 * kBoxBytes;      // one 128 x 128 bf16 key tile
constexpr int64_t kTcMinRows = 4096;                // smaller batches use the SIMT kernels

struct LshTcArgs {
  uint32_t* codes;
  int64_t code_stride;
  int64_t rows;
  int64_t n_tiles;
  int32_t* status;
  uint64_t wait_ns;
};

template <int BITS>
constexpr size_t lsh_tc_smem() {
  return 1024 /* alignment slack */ + (size_t)kTcStages * kTileBytes + (size_t)BITS * 256 + 256;
}

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1)
lsh_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap rmap, LshTcArgs a) {
  constexpr int W = BITS / 32;
  constexpr uint32_t kRBox = BITS * 128;  // one 64-column half of R
  constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kTileRows, BITS);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
  unsigned char* a_s = smem;                                // [stage][2 boxes]
  unsigned char* r_s = smem + kTcStages * kTileBytes;       // [2 boxes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(r_s + 2 * kRBox);
  uint64_t* full = bars;                   // [kTcStages] TMA -> MMA
  uint64_t* empty = bars + kTcStages;      // [kTcStages] MMA -> TMA
  uint64_t* tfull = bars + 2 * kTcStages;  // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;            // [2] epilogue -> MMA
  uint64_t* rfull = tempty + 2;            // R resident
  uint64_t* done = rfull + 1;              // all MMAs of this CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 128);
    }
    tc::mbar_init(rfull, 1);
    tc::mbar_init(done, 1);
    *abort = 0;
    tc::mbar_init_fence();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, 2 * BITS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tc::tma_prefetch_map(&xmap);
    tc::mbar_expect_tx(rfull, 2 * kRBox);
    tc::tma_load_2d(r_s, &rmap, 0, 0, rfull);
    tc::tma_load_2d(r_s + kRBox, &rmap, 64, 0, rfull);
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_phase = 0;  // bit s: stage s armed; parity of its last phase
    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
      if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort, a.wait_ns)) break;
      tc::mbar_expect_tx(&full[stage], kTileBytes);
      const int y = (int)(t * kTileRows);
      tc::tma_load_2d(a_s + stage * kTileBytes, &xmap, 0, y, &full[stage]);
      tc::tma_load_2d(a_s + stage * kTileBytes + kBoxBytes, &xmap, 64, y, &full[stage]);
      armed |= 1u << stage;
      armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == kTcStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // On an abort, let every load already issued land before the CTA leaves.
    if (*abort) {
      for (int s = 0; s < kTcStages; ++s)
        if (armed >> s & 1u) tc::mbar_drain(&full[s], armed_phase >> s & 1u, a.wait_ns);
      tc::mbar_drain(rfull, 0, a.wait_ns);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    bool ok = tc::mbar_wait(rfull, 0, abort, a.wait_ns);
    tc::fence_after_sync();
    const uint32_t r_addr = tc::smem_u32(r_s);
    int stage = 0;
    uint32_t phase = 0;
    int64_t i = 0;
    for (int64_t t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++i) {
      const int acc = (int)(i & 1);
      if (!tc::mbar_wait(&tempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, abort, a.wait_ns)) break;
      if (!tc::mbar_wait(&full[stage], phase, abort, a.wait_ns)) break;
      tc::fence_after_sync();
      const uint32_t a_addr = tc::smem_u32(a_s + stage * kTileBytes);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_bf16(tmem + acc * BITS, tc::sw128_desc(a_addr + kb * kBoxBytes + kk * 32),
                       tc::sw128_desc(r_addr + kb * kRBox + kk * 32), kIdesc, (kb | kk) != 0);
      tc::mma_commit(&empty[stage]);
      tc::mma_commit(&tfull[acc]);
      if (++stage == kTcStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // Every MMA issued above has finished once `done` completes.
    tc::mma_commit(done);
    tc::mbar_drain(done, 0, a.wait_ns);
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row_in_tile = quarter * 32 + lane;
    int64_t i = 0;
    for (int64_t t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++i) {
      const int acc = (int)(i & 1);
      // every lane waits; the warp proceeds only together (tcgen05.ld is warp-wide)
      const bool ok = tc::mbar_wait(&tfull[acc], (uint32_t)((i >> 1) & 1), abort, a.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      uint32_t words[W];
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BITS;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        uint32_t v[32];
        tc::tmem_ld32(taddr + 32 * w, v);
        tc::tmem_wait_ld();
        words[w] = tc::sign_word(v);
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&tempty[acc]);
      const int64_t row = t * kTileRows + row_in_tile;
      if (row < a.rows) {
        uint32_t* dst = a.codes + row * a.code_stride;
        if constexpr (W == 4)
          *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        else
          *reinterpret_cast<uint2*>(dst) = make_uint2(words[0], words[1]);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) report(a.status, HKV_ERR_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_free(tmem, 2 * BITS);
  }
}

// ---- tensor maps (driver entry point, no link-time dependency on libcuda) ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 matrix [rows x 128] with row pitch `pitch_bytes`, read as boxes of
// box_rows x 64 elements with the 128-byte swizzle; rows past the end read 0.
int bf16_rows_map(CUtensorMap* map, const void* base, int64_t rows, int64_t pitch_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return fail(HKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return HKV_OK;
}

template <int BITS>
int run_lsh_tc(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, int32_t* status, cudaStream_t st) {
  alignas(64) CUtensorMap xmap, rmap;
  int rc = bf16_rows_map(&xmap, x, m.rows, m.x_row * 2, kTileRows);
  if (rc == HKV_OK) rc = bf16_rows_map(&rmap, h.R, BITS, kHeadDim * 2, BITS);
  if (rc != HKV_OK) return rc;
  auto kernel = lsh_tc_kernel<BITS>;
  constexpr size_t smem = lsh_tc_smem<BITS>();
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_check(e, "lsh tc smem attribute");
  LshTcArgs args{codes, m.c_row, m.rows, (m.rows + kTileRows - 1) / kTileRows, status, wait_limit_ns()};
  const int64_t grid = args.n_tiles < sm_count() ? args.n_tiles : sm_count();
  kernel<<<(unsigned)grid, kTcThreads, smem, st>>>(xmap, rmap, args);
  return cuda_check(cudaGetLastError(), "lsh tc launch");
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

bool lsh_tc_eligible(const hkv_hash& h, const void* x, const RowMap& m, const uint32_t* codes) {
  const int W = h.code_bits / 32;
  return h.kind == HKV_HASH_LSH && h.dtype == HKV_BF16 && h.head_dim == kHeadDim &&
         (h.code_bits == 64 || h.code_bits == 128) && m.rows >= kTcMinRows && m.per_group == m.rows &&
         m.rows < ((int64_t)1 << 31) && aligned_to(x, 16) && (m.x_row * 2) % 16 == 0 && aligned_to(h.R, 16) &&
         aligned_to(codes, 4 * W) && m.c_row % W == 0;
}

int launch_lsh_tc(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, int32_t* status,
                  cudaStream_t st) {
  return h.code_bits == 128 ? run_lsh_tc<128>(h, x, m, codes, status, st) : run_lsh_tc<64>(h, x, m, codes, status, st);
}

}  // namespace hkv
