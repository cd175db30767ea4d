/*
 * mla_qcache.h -- C ABI of a B200 (sm_100a) library for Multi-Head Latent
 * Attention decode run directly over a low-bit (INT4 / INT2) quantized latent
 * KV cache.
 *
 * What the library computes
 * -------------------------
 * The MLA cache holds, per token, a content latent c (d_c = 512 wide) and a
 * decoupled, already-rotated RoPE key k_r (d_r = 64 wide). QuantMLA
 * (arxivdaily.com/papers/2609.36760, English abstract) stores both paths in
 * low bit widths -- joint INT4, or INT2 content with INT4 RoPE -- and runs a
 * native attention kernel that unpacks and dequantizes inside the attention
 * computation, never materialising a high-precision copy of the history. Decode
 * uses MLA's absorbed MQA form (Group-Query Latent Attention abstract,
 * thelatestinai.com/papers/2607.27269): every head attends the one shared
 * latent with
 *     score_t = (q_c . c_t + q_r . k_r,t) * scale,
 *     o       = sum_t softmax(score)_t * c_t        (latent-space output).
 * The learned transforms of the method are folded into the model weights
 * offline, so none run here; q_c arrives already multiplied by W_UK^T and the
 * output o is consumed by W_UV outside the library.
 *
 * Quantizer (per token, per group of channels, asymmetric round-to-nearest):
 *     s = fp16(fp32(max - min) / (2^bits - 1)),  z = fp16(min),
 *     u = clamp(rint(fp32(x - z) / s), 0, 2^bits - 1)   (u = 0 when s == 0),
 *     x_hat = u * s + z.
 * The arithmetic is IEEE fp32 with round-to-nearest-even, so codes are
 * reproducible bit for bit.
 *
 * Conventions
 * -----------
 *  * The caller owns every buffer (pool, block table, queries, outputs,
 *    workspace). The library allocates no device memory; its only state is
 *    one device status word per GPU (see mla_get_device_status) and the
 *    fixed scratch array of mla_qdecode_noalloc.
 *  * All pointers named "device" must be device memory (or memory the device
 *    can address) of the current CUDA device. "host" pointers are CPU memory.
 *  * Every call that takes a stream is asynchronous on that stream. Argument
 *    errors are detected on the host and returned before anything is
 *    launched. Launch failures return MLA_ERR_CUDA.
 *  * Data found bad on the device (a block-table entry outside [0,num_pages),
 *    a sequence length above the stated maximum) is never dereferenced: the
 *    affected tokens are skipped and the device status word records
 *    MLA_ERR_INVALID_ARG, readable with mla_get_device_status.
 *  * Tensor layouts are row-major and dense unless stated.
 *  * No C++ exception crosses this interface.
 *
 * Page layout (version MLA_QCACHE_LAYOUT_VERSION), per page of page_size
 * tokens, structure of arrays, each segment 16-byte aligned:
 *   [content codes : P x d_c*bits_c/8 B][rope codes : P x d_r*bits_r/8 B]
 *   [content (s,z) : P x d_c/group_c x 4 B][rope (s,z) : P x d_r/group_r x 4 B]
 * Codes are packed little-endian within a byte: channel j of a token's row is
 * at byte j*bits/8, bit (j*bits) mod 8 (for INT4 the even channel is the low
 * nibble). (s,z) are two fp16 values, s at +0 and z at +2. Token t of request
 * b lives in page block_table[b][t / P], slot t % P.
 * Sizes: INT4/INT4 g64 -> 20,736 B per 64-token page (324 B/token, 3.556x
 * smaller than BF16); INT2 g32 content + INT4 g64 RoPE -> 14,592 B (228 B/token,
 * 5.053x).
 */
#ifndef MLA_QCACHE_H
#define MLA_QCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_QCACHE_LAYOUT_VERSION 1

/* A CUDA stream (cudaStream_t). NULL is the legacy default stream. */
typedef struct CUstream_st* mla_stream_t;

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent sizes */
    MLA_ERR_UNSUPPORTED = 2,  /* a shape or bit width this build has no kernel for */
    MLA_ERR_CAPACITY = 3,     /* a sequence would not fit its block-table row */
    MLA_ERR_WORKSPACE = 4,    /* workspace missing, too small or misaligned */
    MLA_ERR_CUDA = 5,         /* a CUDA call failed (no device, launch error) */
    MLA_ERR_TIMEOUT = 6       /* a bounded device-side wait ran out */
} mla_status;

/* Static description of a quantized cache. Supported by this build:
 * d_c = 512, d_r = 64, page_size = 64, bits_c and bits_r in {2, 4},
 * group_c and group_r in {32, 64}. num_pages >= 0 is the pool's page count. */
typedef struct {
    int d_c;
    int d_r;
    int bits_c;
    int group_c;
    int bits_r;
    int group_r;
    int page_size;
    int num_pages;
} mla_qcache_desc;

/* Flags for mla_qdecode / mla_decode_bf16. */
#define MLA_DECODE_DEFAULT 0u
/* Force the CUDA-core (SIMT) kernel instead of the tensor-core kernel; used
 * to cross-check the two. Results agree within the library's error bound. */
#define MLA_DECODE_FORCE_SIMT 1u
/* Skip the compensation terms of the tensor-core kernel (one 16-bit operand
 * per product instead of a hi/lo pair). Faster; its error exceeds the
 * library's stated bound on long, diffuse attention. Never the default. */
#define MLA_DECODE_FAST_UNCOMPENSATED 2u
/* Tests only. The tensor-core decode kernel (s_q * H > 16) never loads its
 * second chunk of keys and every device-side wait gives up after 1 ms, so the
 * call runs the timeout path: the kernel drains and exits, the call returns,
 * mla_get_device_status then reports MLA_ERR_TIMEOUT, and out and lse are
 * undefined. Later calls without the flag are unaffected. Other kernels
 * ignore it. */
#define MLA_DECODE_TEST_STALL 4u

/* Human-readable name of a status code (static storage, never NULL). */
const char* mla_status_string(mla_status s);

/* MLA_QCACHE_LAYOUT_VERSION of the compiled library. */
int mla_qcache_layout_version(void);

/* Check that desc describes a cache this build supports.
 * Returns MLA_OK, MLA_ERR_INVALID_ARG (NULL or impossible values) or
 * MLA_ERR_UNSUPPORTED. Host only; needs no GPU. */
mla_status mla_qcache_check_desc(const mla_qcache_desc* desc);

/* Bytes of one page in the layout above, or 0 if desc is not supported.
 * Host only; needs no GPU. */
size_t mla_qcache_page_bytes(const mla_qcache_desc* desc);

/* Byte offsets of the four page segments: out[0] content codes, out[1] rope
 * codes, out[2] content (s,z), out[3] rope (s,z); out[4] = page bytes.
 * out is host memory with room for 5 values. Host only. */
mla_status mla_qcache_segment_offsets(const mla_qcache_desc* desc, size_t out[5]);

/* Quantize, pack and write new tokens into a paged quantized cache
 * (QuantMLA abstract: the cache is held in INT4 / INT2 and never as a
 * full-history high-precision copy, so tokens are quantized as they are
 * written).
 *   desc              host, a supported description (num_pages = pool pages).
 *   pool              device, num_pages * mla_qcache_page_bytes(desc) bytes,
 *                     256-byte aligned; written in place.
 *   block_table       device int32 [B, max_pages_per_seq]; entries are page
 *                     indices in [0, num_pages).
 *   seq_lens_before   device int32 [B]: tokens already cached per request;
 *                     new token j of request b goes to position
 *                     seq_lens_before[b] + j. The caller updates its lengths.
 *   c_new             device bf16 [B, n_new, d_c], row-major.
 *   kr_new            device bf16 [B, n_new, d_r], already rotated.
 * Values must be finite with |x| <= 65504 (the fp16 range of s and z).
 * B == 0 or n_new == 0 is a no-op that returns MLA_OK.
 * Positions past max_pages_per_seq * page_size, or table entries outside the
 * pool, are skipped and flagged in the device status word. */
mla_status mla_qcache_append(const mla_qcache_desc* desc, void* pool,
                             const int32_t* block_table, int max_pages_per_seq,
                             const int32_t* seq_lens_before,
                             const void* c_new, const void* kr_new,
                             int B, int n_new, mla_stream_t stream);

/* The same for the unquantized comparison cache: pool is device bf16
 * [num_pages, page_size, d_c + d_r] with c in channels [0, d_c) and k_r in
 * [d_c, d_c + d_r). Supports d_c = 512, d_r = 64, page_size = 64. */
mla_status mla_bf16cache_append(void* pool, int num_pages, int page_size,
                                const int32_t* block_table, int max_pages_per_seq,
                                const int32_t* seq_lens_before,
                                const void* c_new, const void* kr_new,
                                int B, int n_new, mla_stream_t stream);

/* Number of key splits the decode calls use for this shape: num_splits if it
 * is > 0 (capped at the page count of max_seq_len), otherwise the library's
 * choice for the current device. 1 means no split and no workspace. Host only
 * (queries the current device's SM count; assumes 148 SMs without a GPU).
 * Returns 0 for arguments no decode accepts (negative sizes, s_q * H > 2^20). */
int mla_decode_num_splits(int B, int s_q, int H, int max_seq_len, int num_splits);

/* Workspace bytes mla_qdecode / mla_decode_bf16 need for this shape and
 * split request (0 when the plan has a single split, and for arguments no
 * decode accepts: B <= 0, negative sizes, s_q * H > 2^20). Host only. */
size_t mla_decode_workspace_bytes(int B, int s_q, int H, int max_seq_len, int num_splits);

/* Low-bit MLA decode in the absorbed MQA form over a quantized paged cache.
 * For request b, query i in [0, s_q) and head h, with
 * L = seq_lens[b] - s_q + 1 + i keys visible (the s_q queries are the last
 * s_q positions, causal among themselves):
 *   out[b,i,h,:] = sum_{t<L} softmax_t(scale*(q_c.c_hat_t + q_r.kr_hat_t)) c_hat_t
 *   lse[b,i,h]   = ln sum_{t<L} exp(scale*(q_c.c_hat_t + q_r.kr_hat_t))
 * where c_hat, kr_hat are the dequantized cache values. Rows with L <= 0
 * give out = 0, lse = -inf.
 *   desc, pool, block_table, max_pages_per_seq: as for mla_qcache_append.
 *   seq_lens      device int32 [B], keys visible to the last query, each
 *                 <= max_seq_len.
 *   max_seq_len   host upper bound on seq_lens; <= max_pages_per_seq*page_size.
 *   q_c           device bf16 [B, s_q, H, d_c]; q_r device bf16 [B, s_q, H, d_r].
 *   scale         softmax scale applied to the sum of both dot products.
 *   num_splits    0 = library choice; > 0 = split each request's keys into
 *                 that many page-aligned chunks merged by a combine kernel.
 *                 Either way no chunk holds more than 8,192 keys (the count
 *                 is raised when needed): the tensor cores' fp32 accumulation
 *                 loses accuracy in proportion to the keys one chunk sums.
 *   workspace     device, >= mla_decode_workspace_bytes(...) bytes, 256-byte
 *                 aligned (may be NULL when that size is 0). Caller-owned
 *                 scratch; contents need no initialisation.
 *   out           device [B, s_q, H, d_c], bf16 (out_dtype 0) or fp32 (1).
 *   lse           device fp32 [B, s_q, H], or NULL.
 *   flags         MLA_DECODE_* bits.
 * Error bound (default flags): max |out - exact| <= 2e-3 * RMS(exact) in fp32
 * output mode, plus half a bf16 ulp of the value in bf16 mode. */
mla_status mla_qdecode(const mla_qcache_desc* desc, const void* pool,
                       const int32_t* block_table, int max_pages_per_seq,
                       const int32_t* seq_lens, int max_seq_len,
                       const void* q_c, const void* q_r,
                       int B, int s_q, int H, float scale, int num_splits,
                       void* workspace, size_t workspace_bytes,
                       void* out, int out_dtype, float* lse,
                       unsigned flags, mla_stream_t stream);

/* One decode step of a speculative-verify / multi-token-prediction loop:
 * the cache append of the step's n_new new tokens followed by mla_qdecode,
 * with the append fused into the decode kernel (the tensor-core kernel, and
 * the small-row kernel for s_q*H <= 16: each work unit quantizes the new
 * tokens inside its key range into the pool, then copies its pages in), which
 * saves the append launch and its latency. Results and pool bytes are those of
 * mla_qcache_append (seq_lens_before = seq_lens - n_new) followed by
 * mla_qdecode; where the fused form does not apply (MLA_DECODE_FORCE_SIMT)
 * the library launches the append kernel and then the decode itself.
 * (QuantMLA abstract: tokens are quantized as they are written; the
 * workload's verify step appends s_q tokens per request before the decode.)
 *   seq_lens      device int32 [B]: lengths AFTER the append; the new tokens
 *                 are positions [seq_lens[b] - n_new, seq_lens[b]). A length
 *                 below n_new is flagged in the device status word and its
 *                 tokens are not written.
 *   c_new, kr_new device bf16 [B, n_new, d_c] and [B, n_new, d_r], 16-byte
 *                 aligned, finite, |x| <= 65504.
 *   n_new         >= 0 (0 makes this exactly mla_qdecode).
 *   pool          device, written in place (the new tokens' slots only).
 *   other arguments as for mla_qdecode. */
mla_status mla_qdecode_fused_append(const mla_qcache_desc* desc, void* pool,
                                    const int32_t* block_table, int max_pages_per_seq,
                                    const int32_t* seq_lens, int max_seq_len,
                                    const void* c_new, const void* kr_new, int n_new,
                                    const void* q_c, const void* q_r,
                                    int B, int s_q, int H, float scale, int num_splits,
                                    void* workspace, size_t workspace_bytes,
                                    void* out, int out_dtype, float* lse,
                                    unsigned flags, mla_stream_t stream);

/* The same decode over the unquantized comparison cache (pool as for
 * mla_bf16cache_append: device bf16 [num_pages, page_size, d_c + d_r]). */
mla_status mla_decode_bf16(const void* pool, int num_pages, int page_size,
                           const int32_t* block_table, int max_pages_per_seq,
                           const int32_t* seq_lens, int max_seq_len,
                           const void* q_c, const void* q_r,
                           int B, int s_q, int H, float scale, int num_splits,
                           void* workspace, size_t workspace_bytes,
                           void* out, int out_dtype, float* lse,
                           unsigned flags, mla_stream_t stream);

/* Scratch held by every GPU that loads this library for mla_qdecode_noalloc. */
#define MLA_QDECODE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* mla_qdecode for callers that cannot allocate device memory when they
 * decode (a serving loop with a fixed memory budget that forbids allocation
 * after start-up, a plug-in whose host framework owns all device memory,
 * latency-critical code where an allocation could synchronise the device).
 * The paper has no counterpart; it is a packaging choice of this library.
 *   Arguments are those of mla_qdecode without the workspace: the split-KV
 *   scratch comes from a fixed array of MLA_QDECODE_NOALLOC_SCRATCH_BYTES
 *   compiled into the library (one per GPU, held until the process exits).
 *   The caller still provides every input and output buffer.
 *   Returns MLA_ERR_WORKSPACE, before launching anything, when the shape
 *   needs more scratch than that (mla_decode_workspace_bytes tells how much);
 *   otherwise the results and errors of mla_qdecode. It calls no allocator.
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.
 *   Every call on a device shares the one array (it keeps the last call's
 *   contents, and nothing in it needs clearing): calls whose executions
 *   overlap on the GPU -- on different streams, or from different host
 *   threads -- race on it and must be serialised by the caller. */
mla_status mla_qdecode_noalloc(const mla_qcache_desc* desc, const void* pool,
                               const int32_t* block_table, int max_pages_per_seq,
                               const int32_t* seq_lens, int max_seq_len,
                               const void* q_c, const void* q_r,
                               int B, int s_q, int H, float scale, int num_splits,
                               void* out, int out_dtype, float* lse,
                               unsigned flags, mla_stream_t stream);

/* ---- Hybrid cache: BF16 protection of the earliest tokens and a recent window ----
 *
 * QuantMLA keeps the earliest tokens and a recent window in BF16 and the
 * history between them in the low-bit cache; history stays visible, only its
 * storage precision differs (QuantMLA podcast episode, the passage on keeping
 * history uncompressed). The pages fix neither sizes nor layout. This library
 * reads them as two caches per request:
 *   protected segment  a BF16 cache (pool and block table as for
 *                      mla_bf16cache_append / mla_decode_bf16) holding the
 *                      sink and the window in position order, newest last;
 *   history            the quantized cache (as for mla_qdecode) holding the
 *                      tokens between them, all older than every query.
 * Tokens enter the window with mla_bf16cache_append and leave it a whole page
 * at a time with mla_qcache_append_bf16_pages; the caller owns both block
 * tables and the page bookkeeping. */

/* Quantize whole BF16 pages into the quantized cache: for each request b with
 * src_pages[b] >= 0, the 64 tokens of page src_pages[b] of bf16_pool are
 * quantized and packed exactly as mla_qcache_append would pack them, and
 * written at positions seq_lens_before[b] .. seq_lens_before[b] + 63 of request
 * b's quantized cache. Requests with src_pages[b] < 0 are skipped.
 *   desc, pool, block_table, max_pages_per_seq, seq_lens_before
 *                     as for mla_qcache_append (device pointers).
 *   bf16_pool         device bf16 [bf16_num_pages, 64, 576], 16-byte aligned.
 *   src_pages         device int32 [B]; entries >= bf16_num_pages are skipped
 *                     and flagged in the device status word.
 * Reads the BF16 pages, writes only the quantized pool. B == 0 is a no-op. */
mla_status mla_qcache_append_bf16_pages(const mla_qcache_desc* desc, void* pool,
                                        const int32_t* block_table, int max_pages_per_seq,
                                        const int32_t* seq_lens_before,
                                        const void* bf16_pool, int bf16_num_pages,
                                        const int32_t* src_pages, int B, mla_stream_t stream);

/* Workspace bytes mla_qdecode_hybrid needs (0 for invalid arguments). */
size_t mla_qdecode_hybrid_workspace_bytes(int B, int s_q, int H, int max_hist_len,
                                          int max_prot_len);

/* Decode over a hybrid cache: one softmax over request b's hist_lens[b]
 * quantized history keys and prot_lens[b] BF16 protected keys. Query i sees
 * every history key and the first prot_lens[b] - s_q + 1 + i protected keys
 * (the protected segment ends with the s_q newest keys, so the window must
 * hold at least s_q tokens). Output and lse as for mla_qdecode.
 *   desc, pool, block_table, max_pages_per_seq
 *                     the quantized history cache (as for mla_qdecode);
 *   hist_lens         device int32 [B], in [0, max_hist_len];
 *   bf16_pool, bf16_num_pages, prot_table, prot_max_pages
 *                     the protected segment's BF16 cache (page size 64);
 *   prot_lens         device int32 [B], in [0, max_prot_len];
 *   q_c, q_r, B, s_q, H, scale, out, out_dtype, lse  as for mla_qdecode;
 *   workspace         device, 256-byte aligned, at least
 *                     mla_qdecode_hybrid_workspace_bytes(...) bytes.
 * The two segments are decoded one after the other (auto split plans) into
 * fp32 partial results in the workspace and merged by log-sum-exp.
 * Errors as for mla_qdecode; MLA_ERR_WORKSPACE if the workspace is short. */
mla_status mla_qdecode_hybrid(const mla_qcache_desc* desc, const void* pool,
                              const int32_t* block_table, int max_pages_per_seq,
                              const int32_t* hist_lens, int max_hist_len,
                              const void* bf16_pool, int bf16_num_pages,
                              const int32_t* prot_table, int prot_max_pages,
                              const int32_t* prot_lens, int max_prot_len,
                              const void* q_c, const void* q_r,
                              int B, int s_q, int H, float scale,
                              void* workspace, size_t workspace_bytes,
                              void* out, int out_dtype, float* lse, mla_stream_t stream);

/* ---- Cache capacity (host arithmetic, no device work) ----
 *
 * Bytes one request of seq_len tokens holds in whole pages: the quantized
 * layout of desc (its num_pages is ignored), or the BF16 cache if desc is NULL
 * (1152 bytes per token). With sink > 0 or window > 0 (desc only), the hybrid
 * policy of mla_qdecode_hybrid as read here: the first `sink` tokens (a whole
 * number of pages) and the newest window .. window + 63 tokens in BF16 pages,
 * the history between them -- 64 * floor((seq_len - sink - window) / 64)
 * tokens -- in quantized pages. Returns 0 for invalid arguments (negative
 * sizes, sink not a multiple of the page size, an unsupported desc). */
size_t mla_cache_bytes_per_request(const mla_qcache_desc* desc, long seq_len, int sink, int window);

/* Largest number of requests of seq_len tokens whose caches fit together in
 * budget_bytes (no page sharing between requests), or -1 for invalid
 * arguments or seq_len == 0 (no bound). The capacity side of the pages' cache-pressure serving result:
 * a format that admits more concurrent requests avoids preemption. */
long mla_cache_max_requests(const mla_qcache_desc* desc, long seq_len, int sink, int window,
                            size_t budget_bytes);

/* Read and clear the current device's status word: waits for `stream`, then
 * stores into *status the first error any kernel recorded since the last
 * read (MLA_OK if none). status is host memory. */
mla_status mla_get_device_status(int* status, mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_QCACHE_H */
