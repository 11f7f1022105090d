// C ABI entry points: argument checks on the host, then launches on the
// caller's stream.  Nothing here allocates device memory or synchronizes,
// except hkv_check.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "internal.h"

namespace hkv {

static thread_local std::string g_last_error;
static std::atomic<int> g_debug_flags{0};
static std::atomic<long long> g_wait_ns{0};
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_check(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return HKV_OK;
  return fail(HKV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

int debug_flags() { return g_debug_flags.load(); }

uint64_t wait_limit_ns() {
  const long long v = g_wait_ns.load();
  return v > 0 ? (uint64_t)v : kDefaultWaitNs;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
  return n;
}

int max_smem_optin() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 48 * 1024;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || n < 1)
    return 48 * 1024;
  return n;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static int check_hash(const hkv_hash* h, bool allow_none = false) {
  if (h == nullptr) return fail(HKV_ERR_INVALID_ARG, "hash is NULL");
  if (allow_none && h->kind == HKV_HASH_NONE) {
    if (h->head_dim != kHeadDim) return fail(HKV_ERR_UNSUPPORTED, "head_dim %d (only 128)", h->head_dim);
    if (h->dtype != HKV_F32 && h->dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", h->dtype);
    if (h->code_bits != 64 && h->code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d", h->code_bits);
    return HKV_OK;
  }
  if (h->head_dim != kHeadDim) return fail(HKV_ERR_UNSUPPORTED, "head_dim %d (only 128)", h->head_dim);
  if (h->dtype != HKV_F32 && h->dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", h->dtype);
  switch (h->kind) {
    case HKV_HASH_LSH:
      if (h->code_bits != 64 && h->code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "LSH code_bits %d (64 or 128)", h->code_bits);
      if (h->R == nullptr) return fail(HKV_ERR_INVALID_ARG, "LSH projection R is NULL");
      break;
    case HKV_HASH_MLP:
      if (h->code_bits != 64 && h->code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "MLP code_bits %d (64 or 128)", h->code_bits);
      if (h->hidden < 1 || h->hidden > 1024) return fail(HKV_ERR_UNSUPPORTED, "MLP hidden %d (1..1024)", h->hidden);
      if (!h->W1 || !h->b1 || !h->W2 || !h->b2) return fail(HKV_ERR_INVALID_ARG, "MLP weight pointer is NULL");
      break;
    case HKV_HASH_SIGN:
      if (h->code_bits != h->head_dim) return fail(HKV_ERR_INVALID_ARG, "SIGN code_bits %d != head_dim", h->code_bits);
      break;
    default:
      return fail(HKV_ERR_INVALID_ARG, "hash kind %d", h->kind);
  }
  return HKV_OK;
}

static int check_heads(int B, int Hq, int Hkv) {
  if (B < 0 || Hq < 1 || Hkv < 1) return fail(HKV_ERR_INVALID_ARG, "B %d Hq %d Hkv %d", B, Hq, Hkv);
  if (Hq % Hkv != 0) return fail(HKV_ERR_INVALID_ARG, "Hq %d not a multiple of Hkv %d", Hq, Hkv);
  if (Hq / Hkv > 16) return fail(HKV_ERR_UNSUPPORTED, "group size %d > 16", Hq / Hkv);
  return HKV_OK;
}

static int check_window(int64_t cap, int64_t N, int n_sink, int n_local, int top_k) {
  if (N < 0 || cap < N) return fail(HKV_ERR_INVALID_ARG, "n_tokens %lld, cap %lld", (long long)N, (long long)cap);
  if (N > INT32_MAX) return fail(HKV_ERR_UNSUPPORTED, "n_tokens %lld > 2^31-1", (long long)N);
  if (n_sink < 0 || n_local < 0 || top_k < 0) return fail(HKV_ERR_INVALID_ARG, "negative sink/local/top_k");
  return HKV_OK;
}

// Workspace of one decode step: [fused scan/select/attend scratch]
// [attention scratch, used when there are no candidates][query codes]
// [selected indices].  Each scratch area keeps its own zero-on-exit invariant.
struct DecodeLayout {
  size_t fused, attend, qcodes, idx, total;
};

static int decode_layout(int B, int Hq, int Hkv, int64_t N, int code_bits, int top_k, int n_sink,
                         int n_local, DecodeLayout& L) {
  RetrieveShape rs{B, Hq, Hkv, code_bits / 32, N, N, n_sink, n_local, top_k};
  AttendShape as{B, Hq, Hkv, HKV_BF16, N, N, top_k, n_sink, n_local};
  const size_t r = retrieve_ws_bytes(rs), d = decode_ws_bytes(rs);
  if ((r == 0 || d == 0) && (int64_t)B * Hkv * top_k > 0) return HKV_ERR_UNSUPPORTED;
  L.fused = align_up(r > d ? r : d, 256);
  L.attend = align_up(attend_ws_bytes(as), 256);
  L.qcodes = align_up(sizeof(uint32_t) * (size_t)B * Hq * (code_bits / 32), 256);
  L.idx = align_up(sizeof(int32_t) * (size_t)B * Hkv * top_k, 256);
  L.total = L.fused + L.attend + L.qcodes + L.idx;
  return HKV_OK;
}

}  // namespace hkv

using namespace hkv;

extern "C" {

const char* hkv_last_error(void) { return g_last_error.c_str(); }

const char* hkv_version(void) { return "hkv 0.1 sm_100a"; }

int hkv_debug_set(int flags, int64_t wait_limit_ns) {
  g_debug_flags.store(flags);
  g_wait_ns.store(wait_limit_ns);
  return HKV_OK;
}

int hkv_check(int32_t* status, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = cuda_check(cudaStreamSynchronize(st), "hkv_check stream sync");
  if (rc != HKV_OK) return rc;
  if (status == nullptr) return HKV_OK;
  int32_t v = 0;
  rc = cuda_check(cudaMemcpyAsync(&v, status, sizeof(v), cudaMemcpyDeviceToHost, st), "hkv_check read");
  if (rc == HKV_OK) rc = cuda_check(cudaMemsetAsync(status, 0, sizeof(int32_t), st), "hkv_check reset");
  if (rc == HKV_OK) rc = cuda_check(cudaStreamSynchronize(st), "hkv_check sync");
  if (rc != HKV_OK) return rc;
  if (v != HKV_OK) fail(v, "device reported status %d", v);
  return v;
}

int hkv_workspace_reset(void* ws, size_t ws_bytes, void* stream) {
  if (ws_bytes == 0) return HKV_OK;
  if (ws == nullptr) return fail(HKV_ERR_INVALID_ARG, "workspace is NULL");
  return cuda_check(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)), "workspace reset");
}

size_t hkv_workspace_bytes(int B, int Hq, int Hkv, int64_t n_tokens, int code_bits, int top_k,
                           int n_sink, int n_local) {
  if (check_heads(B, Hq, Hkv) != HKV_OK || check_window(n_tokens, n_tokens, n_sink, n_local, top_k) != HKV_OK)
    return 0;
  if (code_bits != 64 && code_bits != 128) return 0;
  DecodeLayout L;
  if (decode_layout(B, Hq, Hkv, n_tokens, code_bits, top_k, n_sink, n_local, L) != HKV_OK) return 0;
  return L.total;
}

int hkv_encode_keys(const hkv_hash* hash, const void* x, int64_t rows, int64_t x_stride,
                    uint32_t* codes, int64_t code_stride, uint16_t* norms, int32_t* status,
                    void* stream) {
  int rc = check_hash(hash);
  if (rc != HKV_OK) return rc;
  if (rows < 0) return fail(HKV_ERR_INVALID_ARG, "rows %lld", (long long)rows);
  if (rows == 0) return HKV_OK;
  const int W = hash->code_bits / 32;
  if (!x || !codes) return fail(HKV_ERR_INVALID_ARG, "x or codes is NULL");
  if (x_stride < hash->head_dim || code_stride < W) return fail(HKV_ERR_INVALID_ARG, "stride too small");
  const size_t elt = hash->dtype == HKV_BF16 ? 2 : 4;
  if (!aligned(x, 16) || (x_stride * elt) % 16 != 0) return fail(HKV_ERR_INVALID_ARG, "x rows must be 16-byte aligned");
  if (hash->kind == HKV_HASH_LSH && !aligned(hash->R, 16)) return fail(HKV_ERR_INVALID_ARG, "R must be 16-byte aligned");
  RowMap m{rows, rows, 0, x_stride, 0, code_stride, 0, 1};
  return launch_encode(*hash, x, m, codes, hash->kind == HKV_HASH_SIGN ? norms : nullptr,
                       static_cast<cudaStream_t>(stream), status);
}

size_t hkv_mlp_pack_bytes(int hidden, int code_bits) { return mlp_pack_bytes(hidden, code_bits); }

int hkv_mlp_pack(const hkv_hash* hash, void* packed, size_t packed_bytes, void* stream) {
  int rc = check_hash(hash);
  if (rc != HKV_OK) return rc;
  if (hash->kind != HKV_HASH_MLP) return fail(HKV_ERR_INVALID_ARG, "hkv_mlp_pack needs an MLP hash");
  const size_t need = mlp_pack_bytes(hash->hidden, hash->code_bits);
  if (packed == nullptr || !aligned(packed, 16)) return fail(HKV_ERR_INVALID_ARG, "packed must be 16-byte aligned");
  if (packed_bytes < need) return fail(HKV_ERR_CAPACITY, "packed holds %zu bytes, %zu needed", packed_bytes, need);
  return launch_mlp_pack(*hash, packed, static_cast<cudaStream_t>(stream));
}

int hkv_append(const hkv_hash* hash, int B, int Hkv, int T, const void* k_new, const void* v_new,
               void* K, void* V, uint32_t* codes, uint16_t* norms, int64_t capacity, int64_t pos,
               int32_t* status, void* stream) {
  int rc = check_hash(hash);
  if (rc != HKV_OK) return rc;
  if (B < 0 || Hkv < 1 || T < 0) return fail(HKV_ERR_INVALID_ARG, "B %d Hkv %d T %d", B, Hkv, T);
  if (pos < 0 || pos + T > capacity) return fail(HKV_ERR_CAPACITY, "pos %lld + T %d > capacity %lld", (long long)pos, T, (long long)capacity);
  if (B == 0 || T == 0) return HKV_OK;
  if (!k_new || !v_new || !K || !V || !codes) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(K, 16) || !aligned(V, 16))
    return fail(HKV_ERR_INVALID_ARG, "K/V buffers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t groups = (int64_t)B * Hkv;
  rc = launch_copy_rows(hash->dtype, groups, T, k_new, K, capacity, pos, st);
  if (rc == HKV_OK) rc = launch_copy_rows(hash->dtype, groups, T, v_new, V, capacity, pos, st);
  if (rc != HKV_OK) return rc;
  const int W = hash->code_bits / 32;
  RowMap m{groups * T, T, (int64_t)T * hash->head_dim, hash->head_dim, capacity * W, W, capacity, 1};
  uint16_t* nrm = (hash->kind == HKV_HASH_SIGN && norms) ? norms + pos : nullptr;
  return launch_encode(*hash, k_new, m, codes + pos * W, nrm, st, status);
}

int hkv_retrieve_topk(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                      const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                      int n_local, int top_k, int32_t* idx, int32_t* dist, void* ws,
                      size_t ws_bytes, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!q_codes || !k_codes || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be %d-byte aligned", code_bits / 8);
  RetrieveShape s{B, Hq, Hkv, code_bits / 32, cap, n_tokens, n_sink, n_local, top_k};
  return launch_retrieve(s, q_codes, k_codes, idx, dist, ws, ws_bytes, status, static_cast<cudaStream_t>(stream));
}

int hkv_retrieve_topk_static(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                             const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                             int n_local, int top_k, int32_t* idx, int32_t* dist, int32_t* status,
                             void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!q_codes || !k_codes || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be %d-byte aligned", code_bits / 8);
  RetrieveShape s{B, Hq, Hkv, code_bits / 32, cap, n_tokens, n_sink, n_local, top_k};
  const Window w = window(n_tokens, n_sink, n_local);
  if (w.C == 0)  // nothing to scan: the workspace path only fills idx/dist with -1
    return launch_retrieve(s, q_codes, k_codes, idx, dist, nullptr, 0, status, static_cast<cudaStream_t>(stream));
  return launch_retrieve_static(s, q_codes, k_codes, idx, dist, status, static_cast<cudaStream_t>(stream));
}

int hkv_retrieve_topk_normw(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* k_codes, const uint16_t* norms, int64_t cap, int64_t n_tokens,
                            int n_sink, int n_local, int top_k, int32_t* idx, float* score, void* ws,
                            size_t ws_bytes, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!q_codes || !k_codes || !norms || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be %d-byte aligned", code_bits / 8);
  RetrieveShape s{B, Hq, Hkv, code_bits / 32, cap, n_tokens, n_sink, n_local, top_k};
  return launch_retrieve_normw(s, q_codes, k_codes, norms, idx, score, ws, ws_bytes,
                               static_cast<cudaStream_t>(stream));
}

size_t hkv_normw_workspace_bytes(int B, int Hkv, int64_t n_tokens, int n_sink, int n_local, int top_k) {
  if (B < 0 || Hkv < 1 || check_window(n_tokens, n_tokens, n_sink, n_local, top_k) != HKV_OK) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) return 0;
  const Window w = window(n_tokens, n_sink, n_local);
  return normw_plan(B * Hkv, w.C, top_k, sms).ws_bytes;
}

int hkv_split_select(int G, int rank, int B, int Hq, int Hkv, int code_bits, int top_k, const int32_t* cand_idx,
                     const int32_t* cand_dist, int32_t* idx, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc != HKV_OK) return rc;
  if (G < 1 || rank < 0 || rank >= G || top_k < 0) return fail(HKV_ERR_INVALID_ARG, "G %d rank %d top_k %d", G, rank, top_k);
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!cand_idx || !cand_dist || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if ((int64_t)G * top_k > INT32_MAX) return fail(HKV_ERR_UNSUPPORTED, "G * top_k too large");
  return launch_split_select(G, rank, B * Hkv, top_k, (Hq / Hkv) * code_bits + 1, cand_idx, cand_dist, idx, status,
                             static_cast<cudaStream_t>(stream));
}

int hkv_lse_merge_n(int G, int64_t rows, const float* o, const float* lse, float* out, float* lse_out,
                    void* stream) {
  if (G < 1 || rows < 0) return fail(HKV_ERR_INVALID_ARG, "G %d rows %lld", G, (long long)rows);
  if (rows == 0) return HKV_OK;
  if (!o || !lse || !out) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(o, 16) || !aligned(out, 16)) return fail(HKV_ERR_INVALID_ARG, "o and out must be 16-byte aligned");
  return launch_lse_merge_n(G, rows, o, lse, out, lse_out, static_cast<cudaStream_t>(stream));
}

int hkv_evict_select(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                     const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink, int n_local,
                     int32_t* victim, int32_t* vdist, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, 1);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0) return HKV_OK;
  if (!q_codes || !k_codes || !victim) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be aligned to one code");
  RetrieveShape s{B, Hq, Hkv, code_bits / 32, cap, n_tokens, n_sink, n_local, 1};
  return launch_evict(s, q_codes, k_codes, victim, vdist, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int hkv_write_slots(int B, int Hkv, int dtype, int code_bits, const void* k_new, const void* v_new,
                    const uint32_t* codes_new, const uint16_t* norms_new, void* K, void* V,
                    uint32_t* codes, uint16_t* norms, int64_t capacity, const int32_t* slot,
                    int32_t* status, void* stream) {
  if (B < 0 || Hkv < 1) return fail(HKV_ERR_INVALID_ARG, "B %d Hkv %d", B, Hkv);
  if (dtype != HKV_F32 && dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", dtype);
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (capacity < 1) return fail(HKV_ERR_INVALID_ARG, "capacity %lld", (long long)capacity);
  if (B == 0) return HKV_OK;
  if (!k_new || !v_new || !codes_new || !K || !V || !codes || !slot) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(K, 16) || !aligned(V, 16))
    return fail(HKV_ERR_INVALID_ARG, "K/V rows must be 16-byte aligned");
  return launch_write_slots(dtype, B * Hkv, code_bits / 32, k_new, v_new, codes_new, norms_new, K, V, codes, norms,
                            capacity, slot, status, static_cast<cudaStream_t>(stream));
}

int hkv_sparse_attend(int B, int Hq, int Hkv, int dtype, const void* q, const void* K,
                      const void* V, int64_t cap, int64_t n_tokens, const int32_t* idx,
                      int top_k, int n_sink, int n_local, float scale, float* out, float* lse,
                      void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (dtype != HKV_F32 && dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", dtype);
  if (!std::isfinite(scale)) return fail(HKV_ERR_INVALID_ARG, "scale is not finite");
  if (B == 0) return HKV_OK;
  if (!q || !K || !V || !out || (top_k > 0 && !idx)) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16))
    return fail(HKV_ERR_INVALID_ARG, "q, K, V and out must be 16-byte aligned");
  AttendShape s{B, Hq, Hkv, dtype, cap, n_tokens, top_k, n_sink, n_local};
  return launch_attend(s, q, K, V, idx, scale, out, lse, ws, ws_bytes, status, static_cast<cudaStream_t>(stream));
}

static int check_pages(const int32_t* page_table, int64_t max_pages, int64_t num_pages, int page_size,
                       int64_t n_tokens, PageMap& pm) {
  if (page_size < 1 || max_pages < 0 || num_pages < 1)
    return fail(HKV_ERR_INVALID_ARG, "page_size %d max_pages %lld num_pages %lld", page_size, (long long)max_pages,
                (long long)num_pages);
  if (max_pages * (int64_t)page_size < n_tokens)
    return fail(HKV_ERR_INVALID_ARG, "max_pages * page_size < n_tokens");
  if (n_tokens > 0 && page_table == nullptr) return fail(HKV_ERR_INVALID_ARG, "page_table is NULL");
  pm.table = page_table;
  pm.max_pages = max_pages;
  pm.num_pages = num_pages;
  pm.page_size = page_size;
  return HKV_OK;
}

int hkv_retrieve_topk_paged(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* codes_pool, const int32_t* page_table, int64_t max_pages,
                            int64_t num_pages, int page_size, int64_t n_tokens, int n_sink, int n_local, int top_k,
                            int32_t* idx, int32_t* dist, void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(n_tokens, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  PageMap pm;
  rc = check_pages(page_table, max_pages, num_pages, page_size, n_tokens, pm);
  if (rc != HKV_OK) return rc;
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!q_codes || !codes_pool || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(codes_pool, code_bits / 8))
    return fail(HKV_ERR_INVALID_ARG, "codes_pool must be %d-byte aligned", code_bits / 8);
  if (ws == nullptr) {
    RetrieveShape s{B, Hq, Hkv, code_bits / 32, n_tokens, n_tokens, n_sink, n_local, top_k};
    return launch_retrieve_paged(s, pm, q_codes, codes_pool, idx, dist, status, static_cast<cudaStream_t>(stream));
  }
  // with a workspace: the multi-block scan and selection of hkv_retrieve_topk,
  // reading the codes through the page table
  RetrieveShape s{B, Hq, Hkv, code_bits / 32, n_tokens, n_tokens, n_sink, n_local, top_k, 0, nullptr, &pm};
  return launch_retrieve(s, q_codes, codes_pool, idx, dist, ws, ws_bytes, status, static_cast<cudaStream_t>(stream));
}

int hkv_sparse_attend_paged(int B, int Hq, int Hkv, int dtype, const void* q, const void* K_pool, const void* V_pool,
                            const int32_t* page_table, int64_t max_pages, int64_t num_pages, int page_size,
                            int64_t n_tokens, const int32_t* idx, int top_k, int n_sink, int n_local, float scale,
                            float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(n_tokens, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (dtype != HKV_F32 && dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", dtype);
  if (!std::isfinite(scale)) return fail(HKV_ERR_INVALID_ARG, "scale is not finite");
  PageMap pm;
  rc = check_pages(page_table, max_pages, num_pages, page_size, n_tokens, pm);
  if (rc != HKV_OK) return rc;
  if (B == 0) return HKV_OK;
  if (!q || !K_pool || !V_pool || !out || (top_k > 0 && !idx)) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(q, 16) || !aligned(K_pool, 16) || !aligned(V_pool, 16) || !aligned(out, 16))
    return fail(HKV_ERR_INVALID_ARG, "q, K_pool, V_pool and out must be 16-byte aligned");
  AttendShape s{B, Hq, Hkv, dtype, n_tokens, n_tokens, top_k, n_sink, n_local};
  return launch_attend(s, q, K_pool, V_pool, idx, scale, out, lse, ws, ws_bytes, status,
                       static_cast<cudaStream_t>(stream), &pm);
}

int hkv_lse_merge(int rows, int d, const float* o1, const float* lse1, const float* o2,
                  const float* lse2, float* out, float* lse_out, void* stream) {
  if (rows < 0 || d < 1) return fail(HKV_ERR_INVALID_ARG, "rows %d d %d", rows, d);
  if (rows == 0) return HKV_OK;
  if (!o1 || !lse1 || !o2 || !lse2 || !out) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  return launch_lse_merge(rows, d, o1, lse1, o2, lse2, out, lse_out, static_cast<cudaStream_t>(stream));
}

static int decode_impl(bool per_head, const int32_t* n_tok_b, const hkv_hash* q_hash, int B, int Hq, int Hkv,
                       const void* q,
                    const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                    int64_t n_tokens, int n_sink, int n_local, int top_k, float scale,
                    uint32_t* q_codes, int32_t* idx, float* out, float* lse,
                    const uint32_t* next_k_codes, void* ws, size_t ws_bytes, int32_t* status,
                    void* stream, const PageMap* pm = nullptr) {
  int rc = check_hash(q_hash, true);
  if (rc == HKV_OK) rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (!std::isfinite(scale)) return fail(HKV_ERR_INVALID_ARG, "scale is not finite");
  const bool given_codes = q_hash->kind == HKV_HASH_NONE;
  if (given_codes && q_codes == nullptr) return fail(HKV_ERR_INVALID_ARG, "HKV_HASH_NONE needs q_codes");
  if (B == 0) return HKV_OK;
  if (!q || !k_codes || !K || !V || !out) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) ||
      !aligned(k_codes, q_hash->code_bits / 8) || !aligned(next_k_codes, q_hash->code_bits / 8))
    return fail(HKV_ERR_INVALID_ARG, "q, K, V, out and k_codes must be aligned");
  // selection units: KV heads, or query heads (one index set each)
  const int units = per_head ? Hq : Hkv;
  DecodeLayout L;
  rc = decode_layout(B, Hq, units, n_tokens, q_hash->code_bits, top_k, n_sink, n_local, L);
  if (rc != HKV_OK) return fail(rc, "unsupported decode shape");
  if (ws == nullptr || ws_bytes < L.total) return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, L.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  void* ws_f = base;
  void* ws_a = base + L.fused;
  uint32_t* qc = q_codes ? q_codes : reinterpret_cast<uint32_t*>(base + L.fused + L.attend);
  int32_t* ix = idx ? idx : reinterpret_cast<int32_t*>(base + L.fused + L.attend + L.qcodes);
  const int W = q_hash->code_bits / 32;
  const Window w = window(n_tokens, n_sink, n_local);
  RetrieveShape rs{B, Hq, units, W, cap, n_tokens, n_sink, n_local, top_k, per_head ? Hkv : 0, n_tok_b, pm};
  const bool fused_encode = !given_codes && w.C > 0 && top_k > 0 &&
                            decode_encodes_queries(rs, q_hash->kind, q_hash->dtype);
  if (!given_codes && !fused_encode) {
    RowMap m{(int64_t)B * Hq, (int64_t)B * Hq, 0, q_hash->head_dim, 0, W, 0, 1};
    rc = launch_encode(*q_hash, q, m, qc, nullptr, st, status);
    if (rc != HKV_OK) return rc;
  }
  if (n_tok_b != nullptr && (w.C == 0 || top_k == 0))
    return fail(HKV_ERR_UNSUPPORTED, "ragged decode needs top_k > 0 and n_tokens_max above n_sink + n_local");
  if (w.C == 0 || top_k == 0) {
    // nothing to retrieve: attend the resident rows only
    if (top_k > 0) {
      rc = cuda_check(cudaMemsetAsync(ix, 0xff, sizeof(int32_t) * (size_t)B * units * top_k, st), "idx fill");
      if (rc != HKV_OK) return rc;
    }
    AttendShape as{B, Hq, Hkv, q_hash->dtype, cap, n_tokens, top_k, n_sink, n_local};
    return launch_attend(as, q, K, V, ix, scale, out, lse, ws_a, L.attend, status, st, pm);
  }
  if (fused_encode)
    return launch_decode(rs, q_hash->dtype, q_hash->kind, q_hash->R, nullptr, qc, k_codes, next_k_codes, ix, q, K, V,
                         scale, out, lse, ws_f, L.fused, status, st);
  return launch_decode(rs, q_hash->dtype, HKV_HASH_NONE, nullptr, qc, nullptr, k_codes, next_k_codes, ix, q, K, V,
                       scale, out, lse, ws_f, L.fused, status, st);
}

int hkv_decode_step(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                    const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                    int64_t n_tokens, int n_sink, int n_local, int top_k, float scale,
                    uint32_t* q_codes, int32_t* idx, float* out, float* lse,
                    const uint32_t* next_k_codes, void* ws, size_t ws_bytes, int32_t* status,
                    void* stream) {
  return decode_impl(false, nullptr, q_hash, B, Hq, Hkv, q, k_codes, K, V, cap, n_tokens, n_sink, n_local, top_k,
                     scale, q_codes, idx, out, lse, next_k_codes, ws, ws_bytes, status, stream);
}

int hkv_decode_step_paged(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q, const uint32_t* codes_pool,
                          const void* K_pool, const void* V_pool, const int32_t* page_table, int64_t max_pages,
                          int64_t num_pages, int page_size, int64_t n_tokens, int n_sink, int n_local, int top_k,
                          float scale, uint32_t* q_codes, int32_t* idx, float* out, float* lse, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream) {
  PageMap pm;
  const int rc = check_pages(page_table, max_pages, num_pages, page_size, n_tokens, pm);
  if (rc != HKV_OK) return rc;
  return decode_impl(false, nullptr, q_hash, B, Hq, Hkv, q, codes_pool, K_pool, V_pool, n_tokens, n_tokens, n_sink,
                     n_local, top_k, scale, q_codes, idx, out, lse, nullptr, ws, ws_bytes, status, stream, &pm);
}

int hkv_decode_step_normw(int B, int Hq, int Hkv, int dtype, int code_bits, const void* q, const uint32_t* k_codes,
                          const uint16_t* norms, const void* K, const void* V, int64_t cap, int64_t n_tokens,
                          int n_sink, int n_local, int top_k, float scale, uint32_t* q_codes, int32_t* idx,
                          float* score, float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status,
                          void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (dtype != HKV_F32 && dtype != HKV_BF16) return fail(HKV_ERR_INVALID_ARG, "dtype %d", dtype);
  if (code_bits != kHeadDim) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (sign codes: 128)", code_bits);
  if (B == 0) return HKV_OK;
  if (!q || !k_codes || !norms || !K || !V || !idx || !out) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be %d-byte aligned", code_bits / 8);
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16)) return fail(HKV_ERR_INVALID_ARG, "q, K, V must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const RetrieveShape s{B, Hq, Hkv, code_bits / 32, cap, n_tokens, n_sink, n_local, top_k};
  const Window w = window(n_tokens, n_sink, n_local);
  const int P = B * Hkv;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 1;
  const NormwPlan pl = normw_plan(P, w.C, top_k, sms);
  if (dtype == HKV_BF16 && w.C <= 65536 && (ws == nullptr || pl.nseg == 1))
    return launch_normw_decode(s, q, k_codes, norms, K, V, scale, q_codes, idx, score, out, lse, status, st);
  // query encode, norm-weighted retrieval (segmented with the workspace), attention
  if (q_codes == nullptr) return fail(HKV_ERR_INVALID_ARG, "q_codes is NULL (needed by the multi-launch step)");
  if (ws == nullptr) return fail(HKV_ERR_UNSUPPORTED, "this shape needs a workspace");
  const size_t nw_bytes = align_up(pl.ws_bytes, 256);
  if (ws_bytes < nw_bytes) return fail(HKV_ERR_CAPACITY, "workspace of %zu bytes, %zu needed", ws_bytes, nw_bytes);
  hkv_hash h{};
  h.kind = HKV_HASH_SIGN;
  h.head_dim = kHeadDim;
  h.code_bits = code_bits;
  h.dtype = dtype;
  const int64_t rows = (int64_t)B * Hq;
  RowMap m{rows, rows, 0, kHeadDim, 0, code_bits / 32, 0, 1};
  rc = launch_encode(h, q, m, q_codes, nullptr, st, status);
  if (rc != HKV_OK) return rc;
  rc = launch_retrieve_normw(s, q_codes, k_codes, norms, idx, score, pl.nseg > 1 ? ws : nullptr, nw_bytes, st);
  if (rc != HKV_OK) return rc;
  AttendShape as{B, Hq, Hkv, dtype, cap, n_tokens, top_k, n_sink, n_local};
  return launch_attend(as, q, K, V, idx, scale, out, lse, static_cast<unsigned char*>(ws) + nw_bytes,
                       ws_bytes - nw_bytes, status, st);
}

int hkv_decode_step_heads(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                          const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                          int64_t n_tokens, int n_sink, int n_local, int top_k, float scale,
                          uint32_t* q_codes, int32_t* idx, float* out, float* lse, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream) {
  return decode_impl(true, nullptr, q_hash, B, Hq, Hkv, q, k_codes, K, V, cap, n_tokens, n_sink, n_local, top_k,
                     scale, q_codes, idx, out, lse, nullptr, ws, ws_bytes, status, stream);
}

int hkv_decode_step_ragged(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                           const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                           const int32_t* n_tokens_b, int64_t n_tokens_max, int n_sink, int n_local,
                           int top_k, float scale, uint32_t* q_codes, int32_t* idx, float* out, float* lse,
                           void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  if (n_tokens_b == nullptr) return fail(HKV_ERR_INVALID_ARG, "n_tokens_b is NULL");
  return decode_impl(false, n_tokens_b, q_hash, B, Hq, Hkv, q, k_codes, K, V, cap, n_tokens_max, n_sink, n_local,
                     top_k, scale, q_codes, idx, out, lse, nullptr, ws, ws_bytes, status, stream);
}

int hkv_retrieve_topk_heads(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                            int n_local, int top_k, int32_t* idx, int32_t* dist, void* ws,
                            size_t ws_bytes, int32_t* status, void* stream) {
  int rc = check_heads(B, Hq, Hkv);
  if (rc == HKV_OK) rc = check_window(cap, n_tokens, n_sink, n_local, top_k);
  if (rc != HKV_OK) return rc;
  if (code_bits != 64 && code_bits != 128) return fail(HKV_ERR_UNSUPPORTED, "code_bits %d (64 or 128)", code_bits);
  if (B == 0 || top_k == 0) return HKV_OK;
  if (!q_codes || !k_codes || !idx) return fail(HKV_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned(k_codes, code_bits / 8)) return fail(HKV_ERR_INVALID_ARG, "k_codes must be %d-byte aligned", code_bits / 8);
  RetrieveShape s{B, Hq, Hq, code_bits / 32, cap, n_tokens, n_sink, n_local, top_k, Hkv};
  return launch_retrieve(s, q_codes, k_codes, idx, dist, ws, ws_bytes, status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
