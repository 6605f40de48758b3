/*
 * fa.h -- C ABI of libfa.so: exact scaled-dot-product attention on B200
 * (sm_100a).  A fused forward pass (fixed-length and variable-length) and
 * single-token decode over a paged KV cache.
 *
 * What the calls compute.  Standard attention, as the page "Flash Attention
 * 是什么：2026 最新原理、架构演进与实战详解" (ai.lansai.wang) defines it in its
 * section 核心工作机制: for each query row i,
 *     s_ij = scale * q_i . k_j,    p_ij = exp(s_ij - m_i) / l_i,
 *     o_i  = sum_j p_ij v_j,       lse_i = m_i + ln l_i,
 * with m_i the row max and l_i = sum_j exp(s_ij - m_i).  The forward pass is
 * computed the fused way that page describes (tiling into on-chip blocks,
 * online softmax with a running max and normaliser -- section 关键术语解析,
 * item 4 -- and one final rescale, as the page at zwxr.cn describes in its
 * section 3.1), so the N x N score matrix never reaches device memory.  The
 * same page (section 常见误解澄清, misconception 1) states the result is the
 * standard one up to floating-point rounding; that is the contract here.
 *
 * Conventions shared by every call:
 *  - Element types: q, k, v, o, pages are bf16 (IEEE binary16-brain, raw
 *    uint16 storage); lse is fp32; all index arrays are int32.
 *  - Pointers are DEVICE pointers owned by the caller; the library never
 *    frees or retains them beyond the call's stream work.  Every tensor base
 *    pointer must be 16-byte aligned (FA_ERR_ALIGN otherwise).
 *  - Head dimension d must be 64 or 128 (FA_ERR_UNSUPPORTED otherwise).
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream) and
 *    never synchronise, except fa_get_device_error.  Argument errors are
 *    returned before anything is launched.  FA_ERR_CUDA means a CUDA launch
 *    or runtime call failed (cudaGetLastError is left as CUDA set it).
 *  - Faults found on the device (a bounded wait that ran out, a negative
 *    sequence length) do not trap: the kernel records a code in the library's
 *    device error word and returns; fa_get_device_error reads it.
 *  - The library holds one device workspace per (GPU, stream): the decode
 *    split partials, the rotated K of fa_fwd_rope, the backward pass's
 *    statistics and fp32 dq accumulator, the page offsets of the paged
 *    prefill, append and gather.  It is allocated with cudaMallocAsync on that
 *    stream, grown (freed and reallocated) in the stream's order, and freed by
 *    fa_release_workspace.  So calls on different streams may overlap on the
 *    GPU (e.g. a prefill on one stream and a decode on another); calls on one
 *    stream are ordered by the stream.  The key is the stream handle: destroy
 *    a stream only after its calls have completed (a new stream may get the
 *    same handle), and call fa_release_workspace to return the memory of
 *    streams no longer used.
 *  - Cached device state: the library caches, per GPU, the device addresses
 *    of its error word and of the allocation-free decode's scratch array.
 *    They belong to the GPU's primary context: do not keep using the library
 *    across a cudaDeviceReset (which destroys that context).
 *  - Thread safety: the host entry points may be called from several host
 *    threads; the workspace bookkeeping is guarded by a mutex.
 */
#ifndef FA_H
#define FA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported from libfa.so (which is built with hidden default visibility). */
#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* fa_stream_t;

enum fa_status {
    FA_OK = 0,
    FA_ERR_NULL = -1,           /* a required pointer is NULL */
    FA_ERR_SHAPE = -2,          /* a size is out of range (negative, zero where not allowed, too large) */
    FA_ERR_UNSUPPORTED = -3,    /* d not in {64,128}, page_size != 256, or not an sm_100 device */
    FA_ERR_ALIGN = -4,          /* a tensor base pointer is not 16-byte aligned */
    FA_ERR_CUDA = -5,           /* a CUDA runtime/driver call or launch failed */
    FA_ERR_DEVICE_TIMEOUT = -6, /* reported through fa_get_device_error: a bounded device wait ran out */
    FA_ERR_NOMEM = -7,          /* the library workspace could not be allocated */
    FA_ERR_DEVICE_BAD_INPUT = -8 /* reported through fa_get_device_error: e.g. a negative seq_lens entry */
};

/*
 * fa_fwd -- fused attention forward pass over fixed-length sequences.
 *
 * Computes, for every batch b, head h and query row i < N,
 *   o[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:] . k[b,h,j,:]) v[b,h,j,:]
 *   lse[b,h,i] = natural log of sum_j exp(scale * q[b,h,i,:] . k[b,h,j,:])
 * over keys j < N, or j <= i when `causal` is non-zero (the flash_attn_causal
 * knob of the page "为什么“Flash”突然成了AI圈的高频词" (lqnn.cn), section 3.3,
 * top-left aligned).  `scale` is the softmax scale (that section's
 * softmax_scale; callers normally pass 1/sqrt(d)); any finite value.
 *
 * Layout: q, k, v, o are [B, H, N, d] contiguous bf16 (the [1, 32, 16384, 128]
 * layout of that page's section 2.1); lse is [B, H, N] fp32.
 * Any N >= 1 (no padding to a multiple of the tile is required).
 * Limits: B*H <= 65535, N <= 2^31 - 1 - 128.
 * Returns FA_OK, or an FA_ERR_* code before launching anything.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_fwd_gqa -- fa_fwd with fewer K/V heads than query heads (grouped-query
 * attention; multi-query attention is H_kv = 1).  The page "Flash Attention
 * 是什么" names adapting the fused method to MQA and GQA as the next step
 * (section 进阶学习路径, item 4); the arithmetic per head is fa_fwd's.
 *
 * Query head h reads K/V head h / (H / H_kv):
 *   o[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:] . k[b,g,j,:]) v[b,g,j,:],
 *   g = h / (H / H_kv) (integer division), same mask and lse as fa_fwd.
 * Layout: q, o are [B, H, N, d] bf16; k, v are [B, H_kv, N, d] bf16; lse is
 * [B, H, N] fp32.  H must be a multiple of H_kv (else FA_ERR_SHAPE).
 * fa_fwd is this call with H_kv = H.  Other limits, ownership and errors as
 * fa_fwd.
 */
FA_API int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int H_kv, int N, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_fwd_rope -- fa_fwd_gqa with rotary position embedding fused into the
 * kernel: the page "“Flash”不是那个被时代淘汰的插件" (0539edu.com) describes a
 * kernel that fuses RoPE (section 2) from a precomputed sin/cos lookup table
 * (section 3).  q and k are passed unrotated.  The page applies RoPE with the
 * QKV projection, once per position; here one row-kernel launch rotates Q and
 * K once per position into the library workspace of the call's stream
 * ((B*H + B*H_kv)*N*d*2 bytes, grown on demand), and the forward kernel reads
 * the rotated copies (every query block of a head reads K, so rotating tiles
 * inside the forward kernel would repeat K's rotation once per block).
 *   rope_cos, rope_sin : DEVICE fp32 [max_pos, d/2], row-major; entry (p, i)
 *                        is cos / sin of the angle for position p and pair i
 *                        (normally p * base^(-2i/d)); max_pos >= N
 * Position of row n is n.  Rotate-half pairs: for i < d/2,
 *   x'_i = x_i cos - x_{i+d/2} sin,  x'_{i+d/2} = x_{i+d/2} cos + x_i sin,
 * evaluated in fp32 (each product rounded, then the difference or sum, no
 * fused multiply-add) and rounded to bf16 (the tensor cores' input), then
 * attention as fa_fwd_gqa on the rotated q, k.  Both tables NULL or unaligned:
 * FA_ERR_NULL / FA_ERR_ALIGN; max_pos < N: FA_ERR_SHAPE.
 */
FA_API int fa_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse,
           const float* rope_cos, const float* rope_sin, int max_pos, int B, int H, int H_kv,
           int N, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_bwd -- gradients of fa_fwd (multi-head, fixed length) with respect to
 * q, k and v for an output gradient dout, rebuilding the probabilities from
 * the saved log-sum-exp (the page "Flash Attention 是什么", section
 * 核心工作机制, recomputation paragraph: the forward pass keeps the softmax
 * statistics for the backward pass).
 *   q, k, v, o, dout : [B, H, N, d] bf16 (o as returned by fa_fwd)
 *   lse              : [B, H, N] fp32 as returned by fa_fwd (natural log)
 *   dq, dk, dv       : [B, H, N, d] bf16 outputs
 * With P = exp(scale q k^T - lse) (causal: keys after the query give 0),
 * D_i = dout_i . o_i and dS = P o (dout v^T - D):
 *   dv = P^T dout,   dq = scale dS k,   dk = scale dS^T q.
 * Same `causal`, `scale` and limits as fa_fwd.  Uses the library workspace
 * of the call's stream (B*H*N*(2 + d)*4 bytes: D, the statistics and an fp32
 * dq accumulator), grown on demand.  Accumulation is in fp32; dq sums the
 * contributions of the key blocks with fp32 bulk reduce-adds, so its last
 * bits may differ between runs.
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
           int causal, float scale, fa_stream_t stream);

/*
 * fa_bwd_gqa -- fa_bwd for fa_fwd_gqa: grouped K/V heads (grouped- or
 * multi-query attention, the variants named by the page "Flash Attention
 * 是什么", section 进阶学习路径, item 4).
 *   q, o, dout, dq : [B, H, N, d] bf16;  lse : [B, H, N] fp32
 *   k, v, dk, dv   : [B, H_kv, N, d] bf16 (H a multiple of H_kv, FA_ERR_SHAPE
 *                    otherwise)
 * Query head h uses K/V head h / (H / H_kv); the gradient of a K/V head sums
 * the contributions of every query head of its group (one CTA per K/V head
 * and 128-key block walks the query tiles of all of them).  Everything else
 * as fa_bwd, which is this call with H_kv = H.
 */
FA_API int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                      int H, int H_kv, int N, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_bwd_varlen -- gradients of fa_fwd_varlen (with grouped K/V heads) over
 * B packed sequences of different lengths.
 *   q, o, dout, dq : [total, H, d] bf16;  lse : [H, total] fp32 as returned
 *                    by fa_fwd_varlen
 *   k, v, dk, dv   : [total, H_kv, d] bf16 (H_kv = H for plain multi-head;
 *                    query head h uses K/V head h / (H / H_kv))
 *   cu_seqlens     : DEVICE int32 [B+1], as for fa_fwd_varlen; max_seqlen
 *                    bounds every length (a longer sequence is cut to it and
 *                    reported, like out-of-range offsets)
 * Each sequence's gradients are those of fa_bwd on its own rows.  Workspace:
 * total*H*(2 + d)*4 bytes, as fa_bwd.  Same `causal`, `scale`, d and alignment
 * rules as fa_fwd_varlen.
 */
FA_API int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv,
                         const int32_t* cu_seqlens, int B, int H, int H_kv, int total,
                         int max_seqlen, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_fwd_varlen -- the forward pass over B sequences of different lengths
 * packed back to back (the variable-length batches of the page "Flash
 * Attention 是什么", section 典型应用场景).
 *
 * Sequence b owns packed rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (cu_seqlens
 * is a DEVICE int32 array of B+1 non-decreasing offsets, cu_seqlens[0] = 0).
 * Attention never crosses a sequence; with `causal`, row t of a sequence sees
 * rows 0..t of the same sequence.
 * Layout: q, k, v, o are [total, H, d] bf16; lse is [H, total] fp32.
 * `total` (the packed row count, = cu_seqlens[B]) is passed from the host so
 * that the call never has to read device memory; `max_seqlen` must be >= every
 * sequence length (it sizes the launch).  A cu_seqlens entry that breaks
 * these rules (decreasing, past `total`, a sequence longer than max_seqlen) is
 * clamped on the device and reported as FA_ERR_DEVICE_BAD_INPUT; no access
 * leaves the [total, H, d] tensors.
 */
FA_API int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens, int B, int H, int total, int max_seqlen, int d,
                  int causal, float scale, fa_stream_t stream);

/*
 * fa_fwd_varlen_gqa -- fa_fwd_varlen with grouped K/V heads: q, o
 * [total, H, d], k, v [total, H_kv, d] bf16 (H a multiple of H_kv,
 * FA_ERR_SHAPE otherwise); query head h attends with K/V head h / (H / H_kv)
 * of its own sequence.  fa_fwd_varlen is this call with H_kv = H.
 */
FA_API int fa_fwd_varlen_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                             const int32_t* cu_seqlens, int B, int H, int H_kv, int total,
                             int max_seqlen, int d, int causal, float scale, fa_stream_t stream);

/*
 * fa_decode_paged -- single-token decode over a paged KV cache, split over
 * the cache pages and merged by log-sum-exp.
 *
 * The cache is the fixed-size page pool of the page "“Flash”不是那个被时代淘汰
 * 的插件" (0539edu.com), section 2: every page holds page_size (= 256)
 * consecutive tokens of one sequence.
 *   q          : [B, H, d] bf16, the new token's query of each sequence
 *   k_pages,
 *   v_pages    : [P, H, page_size, d] bf16 -- page p, head h is one contiguous
 *                page_size x d slice
 *   page_table : int32, the pages of all sequences packed back to back:
 *                sequence b's pages are entries off_b .. off_b + n_b - 1 with
 *                n_b = ceil(seq_lens[b] / page_size) and off_b = sum of n over
 *                earlier sequences; token t of sequence b is in page
 *                page_table[off_b + t / page_size], slot t % page_size
 *   seq_lens   : [B] int32, tokens cached per sequence (the new token's k/v
 *                already appended); 0 gives o = 0; a negative entry is treated
 *                as 0 and reported as FA_ERR_DEVICE_BAD_INPUT
 *   o          : [B, H, d] bf16 output
 * The query attends, without a mask, to all seq_lens[b] cached tokens, with
 * softmax scale 1/sqrt(d) (the default of the lqnn.cn page, section 3.3; the
 * call has no scale argument).  page_size must be 256.
 * Uses the library workspace of the call's stream (see the conventions above).
 */
FA_API int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* seq_lens, void* o,
                    int B, int H, int d, int page_size, fa_stream_t stream);

/*
 * fa_decode_paged_gqa -- fa_decode_paged with grouped K/V heads (grouped- or
 * multi-query attention, the variants named by the page "Flash Attention
 * 是什么", section 进阶学习路径, item 4).
 *   q, o       : [B, H, d] bf16
 *   k_pages,
 *   v_pages    : [num_pages, H_kv, page_size, d] bf16 -- the cache holds
 *                H_kv heads
 * Query head h attends to K/V head h / (H / H_kv) of its sequence's cached
 * tokens; everything else (page table, lengths, scale 1/sqrt(d), no mask,
 * workspace) as fa_decode_paged.  Any H that is a multiple of H_kv works;
 * a group of more than 16 query heads (multi-query attention with many
 * heads) runs as equal sub-groups of at most 16, each reading the K/V
 * slices once
 * (FA_ERR_UNSUPPORTED otherwise; FA_ERR_SHAPE if H is not a multiple of
 * H_kv, or num_pages < 1).  Each (page, K/V head) slice is read from device
 * memory once and serves all H / H_kv query heads of its group.  With at
 * most two work units per sequence (a unit is a group, or a pair of 16-head
 * sub-groups: multi-query attention) the tokens of all sequences are
 * divided evenly over the SMs, and the workspace grows with B and the SM
 * count rather than with the sequence lengths.  A page
 * index outside [0, num_pages) is reported as FA_ERR_DEVICE_BAD_INPUT (see
 * fa_get_device_error); nothing outside the pool is read, and the output of
 * that sequence is unspecified.
 */
FA_API int fa_decode_paged_gqa(const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* seq_lens, void* o,
                    int B, int H, int H_kv, int num_pages, int d, int page_size,
                    fa_stream_t stream);

/*
 * fa_decode_paged_strided -- fa_decode_paged_gqa with the page table given
 * as a block table: one fixed-width row of page indices per sequence (the
 * page list each sequence owns in the cache of the page "“Flash”不是那个被
 * 时代淘汰的插件" (0539edu.com), section 2, kept as a [B, max_pages] array,
 * the layout serving engines usually hold).
 *   block_table : [B, max_pages] int32, row-major; sequence b's k-th page is
 *                 block_table[b * max_pages + k]; entries past a sequence's
 *                 ceil(seq_lens[b] / page_size) pages are not read
 *   max_pages   : the row width (>= 1; B * max_pages and
 *                 max_pages * page_size must fit in int32, FA_ERR_SHAPE
 *                 otherwise)
 *   q, k_pages, v_pages, seq_lens, o, B, H, H_kv, num_pages, d, page_size:
 *                 as fa_decode_paged_gqa (H_kv = H for plain multi-head)
 * A length beyond its row (seq_lens[b] > max_pages * page_size) is reported
 * as FA_ERR_DEVICE_BAD_INPUT and decoded over the row's tokens only; no
 * entry outside the table is read.  A first kernel copies the used entries
 * of every row, back to back, into the library workspace of the call's
 * stream (B * max_pages + B int32 beyond the decode's own part), then the decode of
 * fa_decode_paged_gqa runs on that packed table, so results equal
 * fa_decode_paged_gqa's on the same pages bit for bit.
 */
FA_API int fa_decode_paged_strided(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_table, int max_pages,
                                   const int32_t* seq_lens, void* o, int B, int H, int H_kv,
                                   int num_pages, int d, int page_size, fa_stream_t stream);

/*
 * fa_append_paged -- write the K and V rows of new tokens into the paged
 * cache: the step before attention in the serving loop of the page "“Flash”
 * 不是那个被时代淘汰的插件" (0539edu.com), section 2 (a new token goes into a
 * page taken from the fixed pool).
 *   k_new, v_new : [total_new, H_kv, d] bf16, the new rows of all sequences
 *                  packed back to back
 *   cu_new       : DEVICE int32 [B+1], sequence b's new rows are
 *                  cu_new[b] .. cu_new[b+1]-1
 *   k_pages,
 *   v_pages      : [num_pages, H_kv, page_size, d] bf16, updated in place
 *   page_table   : packed as for fa_decode_paged, for the lengths AFTER the
 *                  append; the caller has already taken the pages the new
 *                  tokens need from its free list (page allocation is the
 *                  caller's: the library holds no allocator)
 *   seq_lens     : DEVICE int32 [B], tokens per sequence after the append
 * Sequence b's n_b new rows become its last n_b tokens: new row i goes to
 * position seq_lens[b] - n_b + i, i.e. slot (pos % page_size) of page
 * page_table[off_b + pos / page_size].  page_size must be 256.  A sequence
 * with n_b > seq_lens[b], or a page index outside [0, num_pages), is skipped
 * and reported as FA_ERR_DEVICE_BAD_INPUT (no write leaves the pool).  Uses the
 * library workspace of the call's stream for the page offsets.
 */
FA_API int fa_append_paged(const void* k_new, const void* v_new, const int32_t* cu_new,
                    void* k_pages, void* v_pages, const int32_t* page_table,
                    const int32_t* seq_lens, int B, int H_kv, int total_new, int num_pages,
                    int d, int page_size, fa_stream_t stream);

/*
 * fa_prefill_paged -- attention of several new query tokens per sequence
 * through the paged cache (decode with q_len > 1, or prefill of a chunk that
 * continues cached context), with the forward kernel reading K and V tiles
 * straight from the pages.
 *   q, o       : [total_q, H, d] bf16, sequence b's queries are rows
 *                cu_q[b] .. cu_q[b+1]-1 (cu_q: DEVICE int32 [B+1])
 *   lse        : [H, total_q] fp32
 *   k_pages,
 *   v_pages    : [num_pages, H_kv, 256, d] bf16 (H a multiple of H_kv; query
 *                head h reads K/V head h / (H / H_kv))
 *   page_table,
 *   seq_lens   : as fa_decode_paged; seq_lens[b] counts the cached tokens
 *                INCLUDING the new ones (append them first with
 *                fa_append_paged)
 * Sequence b's q_b = cu_q[b+1] - cu_q[b] queries are its last q_b positions:
 * query i sits at position seq_lens[b] - q_b + i and, with `causal`, attends
 * to the keys at positions up to its own (the mask is aligned to the end of
 * the sequence); without it, to all seq_lens[b] keys.  Softmax scale as
 * fa_fwd.  max_q must be >= every q_b (it sizes the launch).  A sequence with
 * q_b > seq_lens[b] is not computed and is reported as
 * FA_ERR_DEVICE_BAD_INPUT.  Page indices outside [0, num_pages) read zeros.
 * With q_b = 1 and `causal` this is fa_decode_paged for the same cache.
 */
FA_API int fa_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* seq_lens, const int32_t* cu_q,
                    void* o, float* lse, int B, int H, int H_kv, int total_q, int max_q,
                    int num_pages, int d, int page_size, int causal, float scale,
                    fa_stream_t stream);

/*
 * fa_gather_paged -- copy the cached tokens of every sequence out of the page
 * pool into contiguous rows (a checking aid for the decode path's address
 * arithmetic; same page_table / seq_lens conventions as fa_decode_paged).
 *   pages : [P, H, page_size, d] bf16
 *   out   : [sum_b seq_lens[b], H, d] bf16, sequence b starting at row
 *           sum_{b' < b} seq_lens[b']
 * page_size must be 256.  Uses the library workspace of the call's stream.
 */
FA_API int fa_gather_paged(const void* pages, const int32_t* page_table, const int32_t* seq_lens,
                    void* out, int B, int H, int d, int page_size, fa_stream_t stream);

/*
 * fa_decode_paged_noalloc -- the same decode as fa_decode_paged, for callers
 * that must not allocate device memory (the pages have no counterpart: this
 * is a deployment variant of the decode entry point).
 *
 * Who needs it: serving loops that reserve all device memory up front (so
 * that a later allocation can fail, or stall the loop while the allocator
 * synchronises), and host programs with their own device allocator that
 * forbid any other allocation, cannot let the library call cudaMalloc, which
 * fa_decode_paged does on its first call (and whenever it needs a larger
 * workspace).
 *
 * Arguments, layouts and results are those of fa_decode_paged.  The scratch
 * (split offsets and per-split partial outputs) lives in one fixed 16 MiB
 * device array inside the library instead of a workspace; each GPU that
 * loads the library holds it until the process exits.  Nothing is allocated
 * and no allocating routine is called.
 *  - Limit: the partials of at least one split per (sequence, head) must fit,
 *    i.e. roughly 4*B*H*(d+1) bytes <= 16 MiB (B*H <= 32,000 at d = 128);
 *    larger calls return FA_ERR_SHAPE before launching.  Within the limit the
 *    call uses as many splits per sequence (up to fa_decode_paged's) as fit,
 *    so its output can differ from fa_decode_paged's by rounding only.
 *  - The first call on each GPU looks up the array's device address (with
 *    that GPU current) and caches it; make that first call before any stream
 *    capture.
 *  - All calls share the array and it keeps the last call's contents (no part
 *    of it needs to start at zero).  Calls whose kernels overlap on the GPU
 *    race on it: order them on one stream or with events.
 */
FA_API int fa_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* page_table, const int32_t* seq_lens, void* o,
                                   int B, int H, int d, int page_size, fa_stream_t stream);

/*
 * fa_get_device_error -- synchronise `stream`, then read and clear the
 * current GPU's device error word.  *code receives FA_OK or the FA_ERR_*
 * value of the first fault a kernel recorded since the last read.
 * Returns FA_OK, FA_ERR_NULL or FA_ERR_CUDA.
 */
FA_API int fa_get_device_error(int* code, fa_stream_t stream);

/*
 * fa_selftest_bounded_wait -- launch one tiny kernel that waits on a device
 * barrier nothing ever signals, using the same bounded wait as every
 * attention kernel.  The wait gives up after about two seconds and records
 * FA_ERR_DEVICE_TIMEOUT, which fa_get_device_error then returns.  This checks
 * the failure-detection path without hanging or faulting the GPU.
 * Returns FA_OK once launched, or FA_ERR_CUDA.
 */
FA_API int fa_selftest_bounded_wait(fa_stream_t stream);

/*
 * fa_selftest_fwd_stall -- the failure-detection path of the forward kernel
 * itself: fa_fwd (causal, scale 1/sqrt(d), same arguments and layouts) with
 * the K/V copy of ring use `withheld` (0: K of key tile 0, 1: V of tile 0,
 * 2: K of tile 1, ...; every later copy too) never issued, and every wait of
 * the kernel bounded by `wait_us` microseconds (1 .. 2,000,000) instead of
 * the usual two seconds.  In each CTA with that many copies the MMA issuer's
 * wait runs out, records FA_ERR_DEVICE_TIMEOUT and sets the CTA's abort flag;
 * the other roles leave their loops, the copies already started land, the
 * products already issued complete, TMEM is freed and the CTA returns (no
 * trap, no fault: the GPU context stays usable).  o and lse are then partly
 * unwritten.  The page "为什么“Flash”突然成了AI圈的高频词" (lqnn.cn), section 4,
 * reports a kernel that stops on a device-side assertion; this call shows the
 * stall is reported instead.  Returns the status of the launch (as fa_fwd);
 * read the device error with fa_get_device_error.
 */
FA_API int fa_selftest_fwd_stall(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, int withheld, int wait_us, fa_stream_t stream);

/*
 * fa_selftest_decode_stall -- the failure-detection path of the paged decode
 * kernel: fa_decode_paged (same arguments and layouts; page indices are not
 * bounded, as there) with the producer issuing no copy from ring use
 * `withheld` on (ring use u: the K and V slices of the u-th 64-token chunk a
 * CTA streams), and every wait bounded by `wait_us` microseconds (1 ..
 * 2,000,000).  In each CTA with that many chunks the consumers' wait runs
 * out, records FA_ERR_DEVICE_TIMEOUT and sets the CTA's abort flag; the other
 * warps leave their loops, the copies already started land and the CTA
 * returns (no trap, no fault).  o is then unspecified.  Returns the status of
 * the launch; read the device error with fa_get_device_error.
 */
FA_API int fa_selftest_decode_stall(const void* q, const void* k_pages, const void* v_pages,
           const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H, int d,
           int page_size, int withheld, int wait_us, fa_stream_t stream);

/* Free the library workspaces of every stream on the current GPU
 * (synchronises the device first).  Returns FA_OK or FA_ERR_CUDA. */
FA_API int fa_release_workspace(void);

/* A static, human-readable name for a status code. */
FA_API const char* fa_status_str(int status);

/* Library ABI version: 100 * major + minor. */
FA_API int fa_version(void);

/*
 * fa_fwd_set_cta_pairs -- choose the kernel that fa_fwd and fa_fwd_gqa run for
 * d = 128 (process-wide; the results agree within the stated tolerances, not
 * bit for bit).  Zero (the default): one CTA per 256 query rows.  Non-zero:
 * CTA pairs on two SMs share each K/V tile and each product (M = 256 rows
 * across the pair), so every K/V byte leaves L2 once per 512 query rows; it
 * draws less power but waits longer per step (both CTAs' softmax gates each
 * product) and measured slower on B200.  Calls already enqueued are not
 * affected.  Returns the previous setting.  (A tuning control with no
 * counterpart on the pages.)
 */
FA_API int fa_fwd_set_cta_pairs(int enable);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
