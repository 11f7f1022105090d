// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "hkv.h"

namespace hkv {

// Records a printf-style message for hkv_last_error() and returns `code`.
int fail(int code, const char* fmt, ...);
// HKV_ERR_CUDA with the CUDA error string, or HKV_OK for cudaSuccess.
int cuda_check(cudaError_t e, const char* where);

int debug_flags();
uint64_t wait_limit_ns();
int sm_count();
int max_smem_optin();  // opt-in dynamic shared memory per block, bytes

constexpr int kDebugSkipArrive = 1;

// ---- encoders (encode.cu) ----
int launch_encode(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes,
                  uint16_t* norms, cudaStream_t st, int32_t* status = nullptr);
// Tensor-core LSH encoder (encode_tc.cu) for large bf16 batches in one group.
bool lsh_tc_eligible(const hkv_hash& h, const void* x, const RowMap& m, const uint32_t* codes);
int launch_lsh_tc(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, int32_t* status,
                  cudaStream_t st);
// Tensor-core MLP encoder (encode_tc.cu); needs the packed 16-bit weights.
bool mlp_tc_eligible(const hkv_hash& h, const void* x, const RowMap& m, const uint32_t* codes);
int launch_mlp_tc(const hkv_hash& h, const void* x, const RowMap& m, uint32_t* codes, int32_t* status,
                  cudaStream_t st);
size_t mlp_pack_bytes(int hidden, int bits);
int launch_mlp_pack(const hkv_hash& h, void* packed, cudaStream_t st);
int launch_copy_rows(int dtype, int64_t groups, int64_t T, const void* src, void* dst,
                     int64_t dst_group_rows, int64_t dst_row0, cudaStream_t st);

// ---- paged caches ----
// Pool page table[b * max_pages + j] holds tokens [j * page_size,
// (j + 1) * page_size) of sequence b; a page stores [Hkv, page_size, ...].
struct PageMap {
  const int32_t* table = nullptr;
  int64_t max_pages = 0, num_pages = 0;
  int page_size = 0;
};

// ---- retrieval (retrieve.cu) ----
// Hkv is the number of selection units per batch: KV heads (one index set
// per KV head, scored by the sum over its g query heads), or the query heads
// themselves (one index set per query head, kv_heads = the KV heads).
struct RetrieveShape {
  int B, Hq, Hkv, words;
  int64_t cap, N;
  int n_sink, n_local, top_k;
  int kv_heads = 0;  // KV heads of the cache when they differ from Hkv
  const int32_t* n_tok_b = nullptr;  // device [B]: ragged lengths, each <= N (N plans the launch)
  const PageMap* pm = nullptr;       // paged cache: codes, K and V are pools read through pm
};
size_t retrieve_ws_bytes(const RetrieveShape& s);
int launch_retrieve(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                    int32_t* idx, int32_t* dist, void* ws, size_t ws_bytes, int32_t* status,
                    cudaStream_t st);
// hkv_retrieve_topk with the library's fixed scratch instead of a workspace.
constexpr size_t kStaticScratchBytes = (size_t)8 << 20;
int launch_retrieve_static(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                           int32_t* idx, int32_t* dist, int32_t* status, cudaStream_t st);
// Scan + select + attention + merge in one launch (candidates must be
// non-empty).  q_kind HKV_HASH_LSH / HKV_HASH_SIGN: the kernel encodes the
// query heads itself (when decode_encodes_queries says it can) and writes
// them to q_codes_out if non-null; otherwise q_codes_in holds them.
size_t decode_ws_bytes(const RetrieveShape& s);
bool decode_encodes_queries(const RetrieveShape& s, int kind, int dtype);
int launch_decode(const RetrieveShape& s, int dtype, int q_kind, const void* R, const uint32_t* q_codes_in,
                  uint32_t* q_codes_out, const uint32_t* k_codes,
                  const uint32_t* next_codes, int32_t* idx, const void* q, const void* K,
                  const void* V, float scale, float* out, float* lse, void* ws, size_t ws_bytes,
                  int32_t* status, cudaStream_t st);

// ---- eviction (evict.cu) ----
// victim[p] = the candidate with the largest group distance (lowest t on
// ties), -1 without candidates; ws: 8 bytes per pair, zero, returned to zero.
int launch_evict(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes, int32_t* victim,
                 int32_t* vdist, void* ws, size_t ws_bytes, cudaStream_t st);
int launch_write_slots(int dtype, int P, int W, const void* k_new, const void* v_new, const uint32_t* codes_new,
                       const uint16_t* norms_new, void* K, void* V, uint32_t* codes, uint16_t* norms, int64_t cap,
                       const int32_t* slot, int32_t* status, cudaStream_t st);

// ---- norm-weighted sign-VQ retrieval (normw.cu) ----
// Segments per pair of the norm-weighted retrieval; nseg 1 needs no
// workspace (one block per pair, at most 65536 candidates).
struct NormwPlan {
  int nseg = 1;
  int seg_len = 0;   // candidates per segment, a multiple of 4096
  int stride = 0;    // workspace entries per (pair, segment), a multiple of 8
  size_t ws_bytes = 0;
};
NormwPlan normw_plan(int P, int64_t C, int top_k, int sms);
// idx/score [B, Hkv, top_k]; ws nullable (then at most 65536 candidates per pair).
int launch_retrieve_normw(const RetrieveShape& s, const uint32_t* q_codes, const uint32_t* k_codes,
                          const uint16_t* norms, int32_t* idx, float* score, void* ws, size_t ws_bytes,
                          cudaStream_t st);

// ---- token split (split.cu) ----
// cand_idx/cand_dist [G, P, k]; idx_out [P, k]; distances in [0, nbins).
int launch_split_select(int G, int me, int P, int k, int nbins, const int32_t* cand_idx, const int32_t* cand_dist,
                        int32_t* idx_out, int32_t* status, cudaStream_t st);
int launch_lse_merge_n(int G, int64_t rows, const float* o, const float* lse, float* out, float* lse_out,
                       cudaStream_t st);

// ---- paged caches (paged.cu, attend.cu) ----
// Group-Hamming top-k over a paged code pool; up to 65536 candidates per pair.
int launch_retrieve_paged(const RetrieveShape& s, const PageMap& pm, const uint32_t* q_codes,
                          const uint32_t* codes_pool, int32_t* idx, int32_t* dist, int32_t* status, cudaStream_t st);

// ---- attention (attend.cu) ----
struct AttendShape {
  int B, Hq, Hkv, dtype;
  int64_t cap, N;
  int top_k, n_sink, n_local;
};
size_t attend_ws_bytes(const AttendShape& s);
int launch_attend(const AttendShape& s, const void* q, const void* K, const void* V,
                  const int32_t* idx, float scale, float* out, float* lse, void* ws,
                  size_t ws_bytes, int32_t* status, cudaStream_t st, const PageMap* pm = nullptr);
// Norm-weighted sign-VQ decode step in one launch (retrieve.cu): bf16 q, K,
// V; one block per pair, at most 65536 candidates per pair.
int launch_normw_decode(const RetrieveShape& s, const void* q, const uint32_t* k_codes, const uint16_t* norms,
                        const void* K, const void* V, float scale, uint32_t* q_codes, int32_t* idx, float* score,
                        float* out, float* lse, int32_t* status, cudaStream_t st);
// bf16 sparse attention on the fused kernel's tensor-core attention stage
// (retrieve.cu); launch_attend sends bf16 shapes here.
size_t sattend_ws_bytes(const AttendShape& s);
int launch_sattend(const AttendShape& s, const void* q, const void* K, const void* V, const int32_t* idx, float scale,
                   float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status, cudaStream_t st,
                   const PageMap* pm);
int launch_lse_merge(int rows, int d, const float* o1, const float* lse1, const float* o2,
                     const float* lse2, float* out, float* lse_out, cudaStream_t st);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Candidate window shared by retrieval and attention.
struct Window {
  int64_t sink_end, local_start, C;
};
inline Window window(int64_t N, int64_t n_sink, int64_t n_local) {
  Window w;
  w.sink_end = n_sink < N ? n_sink : N;
  int64_t ls = N - n_local;
  w.local_start = ls > w.sink_end ? ls : w.sink_end;
  w.C = w.local_start - w.sink_end;
  return w;
}

}  // namespace hkv
