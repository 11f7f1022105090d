/*
 * hkv.h -- C ABI of the B200 hash-code KV retrieval library.
 *
 * The library implements the decode-time path shared by these pages:
 *   - Spotlight Attention: Towards Efficient LLM Generation via Non-linear
 *     Hashing-based KV Cache Retrieval ("Approach", "Key results"): keys and
 *     queries hashed to short binary codes (sign of a two-layer MLP), top-k
 *     keys retrieved per decode step, exact attention over only those keys,
 *     sink and local-window tokens kept.
 *   - HashEvict: A Pre-Attention KV Cache Eviction Strategy using
 *     Locality-Sensitive Hashing ("Abstract"): codes are signs of Gaussian
 *     projections, scored by Hamming distance against a binary structure
 *     kept in GPU memory, updated at every decoding step.
 *   - Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys
 *     ("Abstract"): sign(k) as a 1-bit code that is both storage and index.
 *   - RetrievalAttention: Accelerating Long-Context LLM Inference via Vector
 *     Retrieval ("Summary", "Approach"): a resident sink/window partial and
 *     the retrieved partial merged by exact log-sum-exp rescaling.
 *
 * Conventions for every entry point:
 *   - Every pointer is a DEVICE pointer owned by the caller, unless stated.
 *     The library keeps no pointer after a call returns and allocates no
 *     device memory; scratch comes from the caller's workspace `ws`.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and never synchronizes, except hkv_check.
 *   - Return value: HKV_OK or a negative hkv_status.  Argument errors are
 *     caught on the host before any launch; hkv_last_error() then describes
 *     the failure (thread-local string, valid until the next call on the
 *     same thread).
 *   - Errors found on the device (an index out of range, a wait that ran out
 *     of time) are written to the caller's int32 status word `status`
 *     (device memory, start at 0): the first error wins, later ones are
 *     dropped.  Read it with hkv_check.
 *   - Layouts are dense row-major with the strides stated.  Codes are uint32
 *     words; bit j of a code is 1 iff the j-th pre-sign value is > 0, stored
 *     in word j / 32 at bit position j % 32.
 *   - The retrieval and decode-step kernels are launched with programmatic
 *     dependent launch: such a launch may be scheduled while the previous
 *     kernel on the stream drains, but it reads and writes nothing in device
 *     memory before that kernel has finished, so stream order holds as usual.
 *   - Sequences in a batch share n_tokens (N), except in the ragged decode
 *     step.  Candidates for retrieval are the tokens [sink_end, local_start)
 *     with sink_end = min(n_sink, N) and local_start = max(sink_end,
 *     N - n_local); sink tokens [0, sink_end) and local tokens
 *     [local_start, N) are always attended.
 */
#ifndef HKV_H
#define HKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HKV_OK = 0,
  HKV_ERR_INVALID_ARG = -1,  /* bad pointer, size, stride or alignment */
  HKV_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. head_dim != 128) */
  HKV_ERR_CAPACITY = -3,     /* pos + T > capacity, or workspace too small */
  HKV_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  HKV_ERR_TIMEOUT = -5,      /* device: a cross-block wait ran out of time */
  HKV_ERR_DEVICE_RANGE = -6  /* device: an index outside [0, n_tokens) was skipped */
} hkv_status;

typedef enum { HKV_F32 = 0, HKV_BF16 = 1 } hkv_dtype;

typedef enum {
  HKV_HASH_LSH = 0,  /* code = sign(R x), R [code_bits, head_dim] Gaussian (HashEvict) */
  HKV_HASH_MLP = 1,  /* code = sign(W2 SiLU(W1 x + b1) + b2) (Spotlight Attention) */
  HKV_HASH_SIGN = 2, /* code = sign(x), code_bits == head_dim (Self-Indexing KVCache) */
  HKV_HASH_NONE = 3  /* hkv_decode_step only: q_codes already holds the query codes */
} hkv_hash_kind;

/* One hash function.  Queries and keys may use different ones (the MLP hash
 * has separate query and key networks).  All pointers are device pointers.
 *   kind       hkv_hash_kind
 *   head_dim   d; 128 is the supported value
 *   code_bits  64 or 128 for LSH and MLP; equal to head_dim for SIGN
 *   hidden     MLP hidden width (1..1024; 512 in the Spotlight setting), 0 otherwise
 *   dtype      hkv_dtype of the hashed vectors x (and of R)
 *   R          LSH: [code_bits, head_dim] in `dtype`, row-major
 *   W1, b1     MLP: [hidden, head_dim], [hidden] fp32
 *   W2, b2     MLP: [code_bits, hidden], [code_bits] fp32
 *   packed     MLP, nullable: the 16-bit copy of W1 and W2 that hkv_mlp_pack
 *              wrote.  With it, large bf16 batches are encoded on the tensor
 *              cores; without it, by the fp32 kernels.
 * For bit-exact agreement with an fp64 reference, R (bf16 inputs) and the MLP
 * weights should hold bf16-representable values and no pre-sign value should
 * lie within 1e-3 of zero. */
typedef struct {
  int32_t kind;
  int32_t head_dim;
  int32_t code_bits;
  int32_t hidden;
  int32_t dtype;
  int32_t reserved;
  const void* R;
  const float* W1;
  const float* b1;
  const float* W2;
  const float* b2;
  const void* packed;
} hkv_hash;

/* Description of the last host-side error on this thread ("" if none). */
const char* hkv_last_error(void);

/* Library version string, e.g. "hkv 0.1 sm_100a". */
const char* hkv_version(void);

/* Synchronizes `stream`, reads the device status word, resets it to 0 and
 * returns the value read (HKV_OK, HKV_ERR_TIMEOUT or HKV_ERR_DEVICE_RANGE),
 * or HKV_ERR_CUDA if the stream reported a CUDA error. */
int hkv_check(int32_t* status, void* stream);

/* Bytes of workspace that hkv_retrieve_topk, hkv_sparse_attend and
 * hkv_decode_step (and their variants) need for this shape on the current
 * device (0 if the shape is invalid or unsupported, or no CUDA device is
 * visible: the plan depends on the device's SM count and shared memory).  The workspace must be zero-filled once before
 * first use (hkv_workspace_reset).  Each call returns the counters and
 * histograms that must start at zero to zero before it ends, including calls
 * that end in a device error, so one workspace serves any number of calls in
 * a row (and CUDA-graph replays).  The layout depends on the shape: before
 * a call of another shape reuses a workspace, zero it again.  Calls that
 * share one workspace must not overlap on the GPU. */
size_t hkv_workspace_bytes(int B, int Hq, int Hkv, int64_t n_tokens, int code_bits, int top_k,
                           int n_sink, int n_local);

/* cudaMemsetAsync(ws, 0, ws_bytes, stream). */
int hkv_workspace_reset(void* ws, size_t ws_bytes, void* stream);

/* Encode `rows` vectors into codes (S1 for keys at prefill, S2 for queries).
 * Spotlight Attention "Approach"; HashEvict "Abstract"; Self-Indexing KVCache
 * "Abstract".
 *   x          rows x head_dim in hash->dtype; row r starts at x + r * x_stride
 *              elements (x_stride >= head_dim; 16-byte aligned rows)
 *   codes      row r written at codes + r * code_stride (uint32 words;
 *              code_stride >= code_bits / 32)
 *   norms      SIGN only, nullable: fp16 bit patterns of ||x_r||_2, row r at
 *              norms[r] (computed in fp64, rounded to nearest even)
 * rows == 0 is a no-op. */
int hkv_encode_keys(const hkv_hash* hash, const void* x, int64_t rows, int64_t x_stride,
                    uint32_t* codes, int64_t code_stride, uint16_t* norms,
                    int32_t* status, void* stream);

/* Bytes of the packed MLP weights for this hidden width and code width:
 * W1 as bf16 [hidden_pad, head_dim] then W2 as fp16 [code_bits, hidden_pad],
 * hidden_pad = hidden rounded up to a multiple of 64 (padding is zero).
 * 0 for an invalid shape. */
size_t hkv_mlp_pack_bytes(int hidden, int code_bits);

/* Writes the packed copy of hash->W1 and hash->W2 (the MLP hash's weights,
 * Spotlight Attention "Approach") into `packed` (device, 16-byte aligned,
 * hkv_mlp_pack_bytes bytes, owned by the caller).  W1 becomes bf16 (exact for
 * bf16-representable weights), W2 fp16 (exact for such weights above 2^-14 in
 * magnitude; smaller ones round to the fp16 subnormal grid, an absolute error
 * below 2^-25).  Set hash->packed to `packed` afterwards; the copy must be
 * redone whenever W1 or W2 change.  Asynchronous on `stream`. */
int hkv_mlp_pack(const hkv_hash* hash, void* packed, size_t packed_bytes, void* stream);

/* Decode-time append (S3; HashEvict "Abstract": the binary structure is
 * updated at every decoding step): copy T new key/value rows per (batch, KV
 * head) into the cache at token positions [pos, pos + T) and encode the new
 * keys into `codes` (and `norms` for SIGN).
 *   k_new, v_new  [B, Hkv, T, head_dim] in hash->dtype
 *   K, V          [B, Hkv, capacity, head_dim] in hash->dtype
 *   codes         [B, Hkv, capacity, code_bits / 32]
 *   norms         SIGN only, nullable: [B, Hkv, capacity] fp16 bits
 * Returns HKV_ERR_CAPACITY if pos < 0 or pos + T > capacity. */
int hkv_append(const hkv_hash* hash, int B, int Hkv, int T, const void* k_new, const void* v_new,
               void* K, void* V, uint32_t* codes, uint16_t* norms, int64_t capacity, int64_t pos,
               int32_t* status, void* stream);

/* Hamming scan + top-k (S4, S5).  HashEvict "Abstract" (Hamming distance of
 * binarized projections); Spotlight Attention "Approach" (top-k retrieval).
 * For KV head j of batch b the score of token t is
 *   D(t) = sum over the g = Hq / Hkv query heads h of that KV head of
 *          popcount(q_code[b, h] XOR k_code[b, j, t]),
 * and the k_eff = min(top_k, candidates) candidates with the smallest D are
 * selected, ties to the lowest t.
 *   q_codes  [B, Hq, code_bits / 32]
 *   k_codes  [B, Hkv, cap, code_bits / 32]; only rows < n_tokens are read
 *   idx      [B, Hkv, top_k] int32: selected tokens in ascending order, then -1
 *   dist     nullable [B, Hkv, top_k] int32: D of each selected token, then -1
 * code_bits is 64 or 128; Hq % Hkv == 0, Hq / Hkv <= 16.  Cross-block waits
 * are bounded; on expiry the status word gets HKV_ERR_TIMEOUT. */
int hkv_retrieve_topk(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                      const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                      int n_local, int top_k, int32_t* idx, int32_t* dist, void* ws,
                      size_t ws_bytes, int32_t* status, void* stream);

/* hkv_retrieve_topk without a workspace argument: the same computation and
 * results, with its scratch taken from a fixed area inside the library.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory -- for example code running inside a
 * serving runtime whose allocator owns every byte of the GPU, or a plugin
 * that is handed buffers but may not call cudaMalloc itself -- and so cannot
 * provide `ws`.
 *   - The scratch is one static device array of 8 MiB, present on every GPU
 *     that loads the library until the process exits.  Shapes whose
 *     hkv_workspace_bytes-style scratch need exceeds 8 MiB are rejected with
 *     HKV_ERR_CAPACITY (the message states the bytes needed).  The retrieval
 *     scratch is nbins * 4 bytes per block plus nbins * 4 + 16 bytes per
 *     (batch, KV head), nbins = g * code_bits + 1, rounded up to 256-byte
 *     pieces.  The number of blocks per (batch, KV head) follows the SM
 *     count, so the need grows with it: on a 148-SM B200, 4 KV heads x 512K
 *     tokens with g = 7 take 37 blocks per KV head, 4 * 37 * 897 * 4 bytes of
 *     per-block counts plus 4 * (897 * 4 + 16) bytes, about 0.52 MiB.
 *   - The first call on a device looks up the array's device address (a
 *     host-side query, cached for the process; do not use this entry point
 *     after a cudaDeviceReset).  Make that first call before any stream
 *     capture.  Every call, the first included, only enqueues work on
 *     `stream`.
 *   - Every call uses the same array and first clears, on `stream`, the
 *     counters and histograms that must start at zero; the rest of the area
 *     is written before it is read.  Calls that overlap on the GPU (other
 *     streams, other host threads) race on the array and must not be issued.
 *   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 * Arguments are those of hkv_retrieve_topk, without ws and ws_bytes. */
int hkv_retrieve_topk_static(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                             const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                             int n_local, int top_k, int32_t* idx, int32_t* dist, int32_t* status,
                             void* stream);

/* hkv_decode_step for a batch of sequences of different lengths: sequence b
 * holds n_tokens_b[b] tokens (device int32 [B], each in [0, n_tokens_max]);
 * its sink, local window and candidates follow from its own length, as for a
 * call with n_tokens = n_tokens_b[b].  n_tokens_max (<= cap) plans the launch
 * and sizes the workspace (hkv_workspace_bytes with n_tokens_max).  A length
 * outside [0, n_tokens_max] is clamped and reported as HKV_ERR_DEVICE_RANGE.
 * top_k must be positive and n_tokens_max > n_sink + n_local (at least one
 * sequence with candidates); HKV_ERR_UNSUPPORTED otherwise. */
int hkv_decode_step_ragged(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                           const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                           const int32_t* n_tokens_b, int64_t n_tokens_max, int n_sink, int n_local,
                           int top_k, float scale, uint32_t* q_codes, int32_t* idx, float* out, float* lse,
                           void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* One index set per query head (RetrievalAttention "Key points": each query
 * head retrieves its own keys).  As hkv_retrieve_topk, but query head h of
 * batch b scores the keys of its KV head j = h / g by its own distance
 *   D_h(t) = popcount(q_code[b, h] XOR k_code[b, j, t])
 * and keeps its own k_eff smallest (ties to the lowest t).
 *   idx, dist  [B, Hq, top_k] (dist nullable)
 * Workspace: hkv_workspace_bytes(B, Hq, Hq, ...) (query heads as the third
 * argument). */
int hkv_retrieve_topk_heads(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink,
                            int n_local, int top_k, int32_t* idx, int32_t* dist, void* ws,
                            size_t ws_bytes, int32_t* status, void* stream);

/* hkv_decode_step with one index set per query head: head h attends over
 * sink + its own selected rows + local rows of KV head h / g.  idx is
 * [B, Hq, top_k]; the workspace as for hkv_retrieve_topk_heads. */
int hkv_decode_step_heads(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                          const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                          int64_t n_tokens, int n_sink, int n_local, int top_k, float scale,
                          uint32_t* q_codes, int32_t* idx, float* out, float* lse, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream);

/* HashEvict eviction (HashEvict "Abstract": at every decoding step the new
 * token's key and value replace the cached token expected to receive the
 * lowest attention, found as the key whose binarized projection is farthest
 * in Hamming distance from the query's).  For KV head j of batch b:
 *   victim[b, j] = the t in [sink_end, local_start) with the largest
 *                  D(t) = sum over the g query heads h of
 *                         popcount(q_code[b, h] XOR k_code[b, j, t]),
 *                  lowest t on ties; -1 when there is no candidate
 *   vdist        nullable [B, Hkv] int32: D(victim), -1 without candidates
 * Sink and local tokens are never evicted.  q_codes, k_codes, cap, n_tokens,
 * n_sink, n_local as for hkv_retrieve_topk.  ws: 8 * B * Hkv bytes, zero
 * before the first call; each call returns it to zero (the first bytes of a
 * hkv_workspace_bytes workspace of the same shape qualify).  Two launches. */
int hkv_evict_select(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                     const uint32_t* k_codes, int64_t cap, int64_t n_tokens, int n_sink, int n_local,
                     int32_t* victim, int32_t* vdist, void* ws, size_t ws_bytes, void* stream);

/* Writes one new token per (batch, KV head) into the cache at position
 * slot[b, j] (e.g. the victim of hkv_evict_select): K and V rows, its code,
 * and its fp16 norm when both norm pointers are given.  slot -1 skips the
 * pair; slot >= capacity skips it and reports HKV_ERR_DEVICE_RANGE.
 *   k_new, v_new  [B, Hkv, head_dim] in dtype;  codes_new [B, Hkv, code_bits/32]
 *   norms_new     nullable [B, Hkv] fp16 bits;  K, V, codes, norms: the cache
 * The new codes come from hkv_encode_keys on k_new. */
int hkv_write_slots(int B, int Hkv, int dtype, int code_bits, const void* k_new, const void* v_new,
                    const uint32_t* codes_new, const uint16_t* norms_new, void* K, void* V,
                    uint32_t* codes, uint16_t* norms, int64_t capacity, const int32_t* slot,
                    int32_t* status, void* stream);

/* Top-k per (batch, KV head) by the norm-weighted sign score.  Self-Indexing
 * KVCache "Abstract": a key's sign code with its norm is its 1-bit vector
 * quantisation.  Reading that pair as the reconstruction |k| sign(k) / sqrt(b)
 * and each query head as sign(q_h) / sqrt(b), the inner products summed over
 * the g query heads of KV head j give the score
 *   S(t) = norm[b, j, t] * (g * code_bits - 2 * D(t)),
 *   D(t) = sum_h popcount(q_codes[b, h] XOR k_codes[b, j, t]),
 * and the top_k candidates t in [sink_end, local_start) with the LARGEST S
 * are kept, ties to the lowest t, in ascending t order (-1 past
 * k_eff = min(top_k, candidates)).  S is exact in fp32 (fp16 norm times an
 * integer of at most 12 bits); -0 and +0 are one score.
 *   q_codes [B, Hq, code_bits/32];  k_codes [B, Hkv, cap, code_bits/32]
 *   norms   [B, Hkv, cap] fp16 bits (finite), e.g. from hkv_encode_keys
 *           with the sign hash
 *   idx     [B, Hkv, top_k] int32 out;  score  nullable [B, Hkv, top_k]
 *           fp32 out (S of each selected token, -inf past k_eff)
 * ws nullable.  Without a workspace: one launch, one block per (batch, KV
 * head), at most 65536 candidates per KV head (HKV_ERR_UNSUPPORTED beyond).
 * With one of hkv_normw_workspace_bytes bytes (16-byte aligned; no zero
 * fill needed; HKV_ERR_CAPACITY if smaller): when that size is non-zero,
 * each KV head's window is cut into segments of at most 65536 candidates
 * (enough of them to fill the GPU when there are few KV heads), one block
 * per segment keeps the segment's own top_k in the workspace, and a second
 * launch, one block per KV head, selects the top_k among those lists.  The
 * result is the same either way.  The selected rows go to
 * hkv_sparse_attend like those of hkv_retrieve_topk. */
int hkv_retrieve_topk_normw(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* k_codes, const uint16_t* norms, int64_t cap, int64_t n_tokens,
                            int n_sink, int n_local, int top_k, int32_t* idx, float* score, void* ws,
                            size_t ws_bytes, void* stream);

/* Norm-weighted sign-VQ decode step (Self-Indexing KVCache, "Abstract";
 * Spotlight Attention "Approach"; RetrievalAttention "Approach"): the sign
 * codes of the query heads, the top_k of each KV head by the norm-weighted
 * score (exactly as hkv_retrieve_topk_normw), then the attention of its g
 * query heads over the selected, sink and local rows, merged into out / lse.
 *   dtype   HKV_BF16 or HKV_F32 (q, K, V)
 *   code_bits 128 (the sign of each of the 128 dimensions)
 *   q       [B, Hq, 128];  k_codes [B, Hkv, cap, 4] (sign codes)
 *   norms   [B, Hkv, cap] fp16 bits;  K, V [B, Hkv, cap, 128]
 *   q_codes [B, Hq, W] out, nullable on the one-launch path
 *   idx     [B, Hkv, top_k] int32 out (required; ascending, -1 padded)
 *   score   nullable fp32 out as in hkv_retrieve_topk_normw
 *   out     [B, Hq, 128] fp32;  lse nullable [B, Hq] fp32
 * bf16 windows of at most 65536 candidates run in one launch (one block per
 * KV head: query codes by ballots, the selection, then the tensor-core
 * attention) when ws is NULL or hkv_normw_workspace_bytes(...) is 0.  Any
 * other shape runs query encode + norm-weighted retrieval + sparse
 * attention; ws then holds hkv_normw_workspace_bytes(...) bytes rounded up to
 * a multiple of 256, followed by hkv_workspace_bytes(...) bytes zero-filled
 * once (hkv_workspace_reset), and q_codes is required. */
int hkv_decode_step_normw(int B, int Hq, int Hkv, int dtype, int code_bits, const void* q, const uint32_t* k_codes,
                          const uint16_t* norms, const void* K, const void* V, int64_t cap, int64_t n_tokens,
                          int n_sink, int n_local, int top_k, float scale, uint32_t* q_codes, int32_t* idx,
                          float* score, float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status,
                          void* stream);

/* Workspace bytes of hkv_retrieve_topk_normw for this shape on the current
 * device: 0 when one block per KV head is the plan (no workspace needed),
 * and 0 if the shape is invalid or no CUDA device is visible (the plan
 * depends on the SM count). */
size_t hkv_normw_workspace_bytes(int B, int Hkv, int64_t n_tokens, int n_sink, int n_local, int top_k);

/* Token-split selection.  One sequence's cache is cut into G contiguous
 * token ranges, one per rank, in token order.  Every rank first takes its
 * own top_k with hkv_retrieve_topk over its range (local indices and
 * distances, -1 past its own k_eff); every token of the whole sequence's
 * top_k is among them.  Given all ranks' candidates, gathered rank-major,
 *   cand_idx, cand_dist  [G, B, Hkv, top_k] int32,
 * this call finds the whole sequence's top_k (smallest group distance, ties
 * to the lowest token index: rank order, then ascending local index) and
 * writes the selected tokens of rank `rank` as its local indices:
 *   idx  [B, Hkv, top_k] int32 out, ascending, -1 padded.
 * These are exactly the tokens of that range which hkv_retrieve_topk over
 * the whole sequence would select.  RetrievalAttention "Approach" (retrieval
 * spread over several index partitions, results merged).  A distance
 * outside [0, g * code_bits] is skipped and reported as
 * HKV_ERR_DEVICE_RANGE.  One launch; no workspace. */
int hkv_split_select(int G, int rank, int B, int Hq, int Hkv, int code_bits, int top_k, const int32_t* cand_idx,
                     const int32_t* cand_dist, int32_t* idx, int32_t* status, void* stream);

/* G-way log-sum-exp merge of partial attention results (RetrievalAttention
 * "Approach"), e.g. one partial per rank of a token split.  Per row:
 *   M = max_g lse[g], w_g = exp(lse[g] - M)
 *   out = sum_g w_g o[g] / sum_g w_g,  lse_out = M + log sum_g w_g
 * Rows whose partials are all empty (lse -inf) give out 0, lse_out -inf.
 *   o [G, rows, 128] fp32 (16-byte aligned);  lse [G, rows] fp32
 *   out [rows, 128] fp32;  lse_out nullable [rows] fp32 */
int hkv_lse_merge_n(int G, int64_t rows, const float* o, const float* lse, float* out, float* lse_out,
                    void* stream);

/* Sparse attention over sink + selected + local rows, with the log-sum-exp
 * merge of the partials (S6, S7, S8).  Spotlight Attention "Approach" (exact
 * attention over the retrieved tokens); RetrievalAttention "Approach" (exact
 * log-sum-exp rescaling of partial attention).
 * For query head h (KV head j = h / g):
 *   out[b, h] = sum_t softmax_t(scale * q[b, h] . K[b, j, t]) V[b, j, t]
 *   lse[b, h] = log sum_t exp(scale * q[b, h] . K[b, j, t])
 * over t in [0, sink_end) + {idx[b, j, i] >= 0} + [local_start, n_tokens).
 *   q       [B, Hq, 128] in dtype;  K, V  [B, Hkv, cap, 128] in dtype
 *   idx     [B, Hkv, top_k] int32 (negative entries, e.g. the -1 padding,
 *           are skipped; entries at or past n_tokens are skipped and reported
 *           as HKV_ERR_DEVICE_RANGE)
 * bf16: the fused decode kernel's tensor-core attention stage, a pair's rows
 * split over up to one wave of blocks (cooperative launch) and merged by its
 * last blocks; fp32: a SIMT kernel, split-K with a last-block merge.
 *   out     [B, Hq, 128] fp32;  lse  nullable [B, Hq] fp32
 * The selected indices must not repeat a sink or local token. */
int hkv_sparse_attend(int B, int Hq, int Hkv, int dtype, const void* q, const void* K,
                      const void* V, int64_t cap, int64_t n_tokens, const int32_t* idx,
                      int top_k, int n_sink, int n_local, float scale, float* out, float* lse,
                      void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* Paged cache.  Each sequence's cache is cut into pages of page_size tokens
 * held anywhere in one pool; page_table[b, j] (device int32 [B, max_pages])
 * names the pool page holding tokens [j * page_size, (j + 1) * page_size) of
 * sequence b, and a page stores all KV heads of its tokens:
 *   codes_pool [num_pages, Hkv, page_size, code_bits/32] uint32
 *   K_pool, V_pool [num_pages, Hkv, page_size, 128] in dtype
 * (hkv_encode_keys on the pool viewed as [num_pages * Hkv * page_size, 128]
 * rows fills codes_pool).  The two calls below compute exactly what
 * hkv_retrieve_topk and hkv_sparse_attend compute on the same tokens stored
 * contiguously; only the addressing differs.  The paged layout is this
 * library's storage choice, not the pages' method.  Requirements:
 * page_size >= 1, max_pages * page_size >= n_tokens, num_pages >= 1.  A
 * page id outside [0, num_pages) met on the device is reported as
 * HKV_ERR_DEVICE_RANGE: retrieval gives its tokens the largest distance and
 * attention skips them.
 *
 * Retrieval: idx [B, Hkv, top_k] int32 and nullable dist, as
 * hkv_retrieve_topk.  ws nullable: without a workspace, one block per
 * (batch, KV head) and at most 65536 candidates per KV head
 * (HKV_ERR_UNSUPPORTED beyond); with one (hkv_workspace_bytes of the same
 * shape, zeroed once, as hkv_retrieve_topk's), the multi-block scan and
 * selection of hkv_retrieve_topk at any length. */
int hkv_retrieve_topk_paged(int B, int Hq, int Hkv, int code_bits, const uint32_t* q_codes,
                            const uint32_t* codes_pool, const int32_t* page_table, int64_t max_pages,
                            int64_t num_pages, int page_size, int64_t n_tokens, int n_sink, int n_local, int top_k,
                            int32_t* idx, int32_t* dist, void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* hkv_decode_step over a paged cache: the same computation (query encode,
 * retrieval, attention over the selected and resident rows, merge), with the
 * codes, K and V read through the page table from pools laid out as above
 * (codes_pool, K_pool, V_pool), the sequence length n_tokens <= max_pages *
 * page_size, and the workspace of hkv_workspace_bytes(B, Hq, Hkv, n_tokens,
 * ...).  A page id outside the pool is reported as HKV_ERR_DEVICE_RANGE; its
 * tokens get the largest distance and are not attended. */
int hkv_decode_step_paged(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q, const uint32_t* codes_pool,
                          const void* K_pool, const void* V_pool, const int32_t* page_table, int64_t max_pages,
                          int64_t num_pages, int page_size, int64_t n_tokens, int n_sink, int n_local, int top_k,
                          float scale, uint32_t* q_codes, int32_t* idx, float* out, float* lse, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream);

/* Attention over a paged cache: hkv_sparse_attend with K and V read through
 * the page table (q, idx, out, lse, scale, ws as there; the workspace size
 * is the same). */
int hkv_sparse_attend_paged(int B, int Hq, int Hkv, int dtype, const void* q, const void* K_pool, const void* V_pool,
                            const int32_t* page_table, int64_t max_pages, int64_t num_pages, int page_size,
                            int64_t n_tokens, const int32_t* idx, int top_k, int n_sink, int n_local, float scale,
                            float* out, float* lse, void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* Elementwise log-sum-exp merge of two partial attention results (S8 alone).
 * RetrievalAttention "Approach".  For each of `rows` rows:
 *   m = max(lse1, lse2), w_i = exp(lse_i - m)
 *   out = (w1 o1 + w2 o2) / (w1 + w2), lse_out = m + log(w1 + w2)
 * A part with lse = -inf is empty; two empty parts give out = 0, lse = -inf.
 *   o1, o2, out  [rows, d] fp32;  lse1, lse2, lse_out  [rows] fp32 */
int hkv_lse_merge(int rows, int d, const float* o1, const float* lse1, const float* o2,
                  const float* lse2, float* out, float* lse_out, void* stream);

/* One whole decode step (S2, S4-S8): one kernel that encodes the query heads
 * (LSH, sign), scans, selects, attends and merges; the MLP query hash adds one
 * launch before it.  Results equal hkv_encode_keys on q, then
 * hkv_retrieve_topk, then hkv_sparse_attend: q_codes and idx bit-identical,
 * out and lse within floating-point rounding.
 *   q_hash   hash for the queries (q_hash->dtype is the dtype of q, K, V).  With
 *            kind HKV_HASH_NONE nothing is encoded: q_codes is an input that
 *            already holds the query codes
 *   q        [B, Hq, 128];  k_codes [B, Hkv, cap, code_bits / 32]
 *   K, V     [B, Hkv, cap, 128]
 *   q_codes  [B, Hq, code_bits / 32]: output (nullable) or, for HKV_HASH_NONE,
 *            input (required)
 *   idx      nullable [B, Hkv, top_k] out
 *   out      [B, Hq, 128] fp32;  lse nullable [B, Hq] fp32
 *   next_k_codes  nullable hint: the key codes the next call on this stream
 *            will scan (same shape, e.g. the next layer's).  After its own
 *            scan the kernel asks L2 to prefetch them, so that stream overlaps
 *            this call's selection and attention.  Never read otherwise; the
 *            results do not depend on it. */
int hkv_decode_step(const hkv_hash* q_hash, int B, int Hq, int Hkv, const void* q,
                    const uint32_t* k_codes, const void* K, const void* V, int64_t cap,
                    int64_t n_tokens, int n_sink, int n_local, int top_k, float scale,
                    uint32_t* q_codes, int32_t* idx, float* out, float* lse, const uint32_t* next_k_codes, void* ws,
                    size_t ws_bytes, int32_t* status, void* stream);

/* Testing aid (process-wide).  flags bit 0: in the next retrieval launches,
 * block 0 does not signal its arrival at the cross-block wait, so the wait
 * runs out and reports HKV_ERR_TIMEOUT.  wait_limit_ns: limit of every
 * cross-block wait (0 restores the default of 2 s). */
int hkv_debug_set(int flags, int64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* HKV_H */
