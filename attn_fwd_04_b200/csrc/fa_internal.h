// fa_internal.h -- constants and launch entry points shared inside libfa.so.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"

// A bounded device wait gives up after this much global time.
#define FA_WAIT_TIMEOUT_NS 2000000000ull

// Values written to the device error word: the magnitude of the FA_ERR_*
// status the host reports for them.
#define FA_DEVERR_TIMEOUT (static_cast<unsigned int>(-FA_ERR_DEVICE_TIMEOUT))
#define FA_DEVERR_BAD_INPUT (static_cast<unsigned int>(-FA_ERR_DEVICE_BAD_INPUT))

namespace fa {

// ---- forward -------------------------------------------------------------
struct FwdParams {
    // tensor maps live in the kernel's parameter space (see the launchers)
    void* o;             // bf16 output
    float* lse;          // fp32 output
    const int32_t* cu_seqlens;  // varlen only
    int B, H, N;         // N: sequence length (fixed) or max_seqlen (varlen)
    int H_kv;            // K/V heads; query head h reads K/V head h / (H / H_kv)
    const int32_t* page_table;  // paged prefill: packed page table
    const int32_t* ctx_lens;    // paged prefill: cached tokens (keys) per sequence
    int total;           // varlen: packed rows
    int causal;
    float scale_log2;    // scale * log2(e)
    unsigned int* err;   // device error word
    // packed sequences: the sequences in the order their CTAs run, heaviest
    // first (launch_seq_order; paged prefill); null: 0, 1, ..., B-1
    const int32_t* seq_order;
    // failure-detection check only (fa_selftest_fwd_stall; 0 in every other call):
    uint64_t wait_ns;    // bound of every wait in the kernel (0: FA_WAIT_TIMEOUT_NS)
    int withhold_copy;   // 1 + the K/V ring use whose copy the producer withholds (0: none)
};

// rotary embedding of x0 [rows0, N, d] into y0 and x1 [rows1, N, d] into y1
// (positions 0..N-1), one launch
int launch_rope_rows(const void* x0, void* y0, int64_t rows0, const void* x1, void* y1,
                     int64_t rows1, const float* cos_t, const float* sin_t, int N, int d,
                     int num_sms, cudaStream_t stream);
// forward modes; kFixedPair: fixed length on CTA pairs (2-SM products; d = 128,
// no RoPE), its K map with 64 x 64 boxes (tq, tv: 64 x 128 as for kFixed)
constexpr int kFixed = 0, kVarlen = 1, kPaged = 2, kFixedPair = 3;
int launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, int d, int mode, cudaStream_t stream);
// order[0..B) <- the packed sequences sorted by the forward pass's work on
// them, heaviest first (ties by index): query rows from cu_seqlens, keys from
// ctx_lens (paged prefill, the queries ending the sequence) or the rows
// themselves.  Up to kSeqOrderMax sequences (more: leave the order alone).
constexpr int kSeqOrderMax = 4096;
int launch_seq_order(const int32_t* cu_seqlens, const int32_t* ctx_lens, int B, int causal,
                     int32_t* order, cudaStream_t stream);

// ---- backward ------------------------------------------------------------
size_t bwd_workspace_bytes(int B, int H, int N, int d);
size_t bwd_dq_acc_offset(int B, int H, int N);  // fp32 dQ accumulator, in the workspace
int launch_bwd(const void* o, const void* dout, const float* lse, void* dq, void* dk, void* dv,
               const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& tdo, const CUtensorMap& tdq, int B, int H, int H_kv, int N, int d,
               int causal, float scale, void* workspace, unsigned int* err, int num_sms,
               cudaStream_t stream, const int32_t* cu_seqlens = nullptr, int total = 0);

// ---- paged decode ----------------------------------------------------------
// Number of pages a split covers at least (a split is one CTA work unit) and
// the most splits one sequence is cut into.  With at least kDecodeManyUnits
// units per split (K/V heads, or sub-groups of large groups), 4 pages measured
// fastest on the paged-decode workload for 32 and 8 K/V heads (2: 2-3 %
// slower, more partials and per-unit combines; 8: a longer tail).  With fewer
// units per split the launch is short and 6 pages measured faster (4 K/V
// heads: 6486-6518 GB/s against 6253-6296 with 4 pages; 8 pages 1 % slower).
// The grouped decode with one or two units per split does not cut splits:
// it divides the chunk stream evenly over the CTAs.
constexpr int kDecodeChunkPages = 4;
constexpr int kDecodeChunkPagesFew = 6;
constexpr int kDecodeManyUnits = 8;
constexpr int kDecodeMaxSplits = 64;

struct DecodePlan {
    int32_t* page_off;   // [B+1] prefix of pages per sequence
    int32_t* tok_off;    // [B+1] prefix of tokens per sequence
    int32_t* unit_off;   // [B+1] prefix of (split x head) units per sequence
};

size_t decode_workspace_bytes(int B, int H, int d, int max_splits);
// the grouped decode's workspace (H > Hk): a balanced partition over
// num_sms CTAs for few unit heads, split units otherwise
size_t decode_gqa_workspace_bytes(int B, int H, int Hk, int d, int max_splits, int num_sms);

// H query heads over Hk K/V heads (any H % Hk == 0).  The grouped
// kernels (H > Hk) read the pool through tk, tv: (d, 256, num_pages * Hk)
// maps with 64 x 64 x 1 boxes and 128-byte swizzle and need
// decode_gqa_workspace_bytes of workspace (workspace_bytes is checked); H == Hk reads it with bulk copies, takes no
// maps (may be null) and needs decode_workspace_bytes(B, H, d, max_splits).
// Page indices outside [0, num_pages) are reported.
int launch_decode(const void* q, const void* k_pages, const void* v_pages,
                  const CUtensorMap* tk, const CUtensorMap* tv, const int32_t* page_table,
                  const int32_t* seq_lens, void* o, int B, int H, int Hk, int num_pages, int d,
                  int page_size, int max_splits, void* workspace, size_t workspace_bytes,
                  unsigned int* err, int num_sms, cudaStream_t stream);
bool decode_group_supported(int H, int Hk);
// The multi-head decode with the failure-detection check's settings: every
// wait bounded by wait_ns, and the producer stops issuing copies at ring use
// withhold - 1 (workspace: decode_workspace_bytes(B, H, d, kDecodeMaxSplits)).
int launch_decode_stall(const void* q, const void* k_pages, const void* v_pages,
                        const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                        int d, int page_size, void* workspace, unsigned int* err, int num_sms,
                        cudaStream_t stream, uint64_t wait_ns, int withhold);

// Block table [B, max_pages] -> packed table `packed` (at most B * max_pages
// entries) and lengths `lens` [B] cut to each row, for launch_decode.
int launch_decode_pack(const int32_t* block_table, int max_pages, const int32_t* seq_lens, int B,
                       int page_size, int32_t* packed, int32_t* lens, unsigned int* err,
                       cudaStream_t stream);

// The current device's error word and SM count (sm_100 devices only).
int device_error_word(unsigned int** err, int* num_sms);

int launch_append(const void* k_new, const void* v_new, const int32_t* cu_new, void* k_pages,
                  void* v_pages, const int32_t* page_table, const int32_t* seq_lens, int B,
                  int Hk, int total_new, int d, int page_size, int num_pages, void* workspace,
                  unsigned int* err, int num_sms, cudaStream_t stream);

int launch_gather(const void* pages, const int32_t* page_table, const int32_t* seq_lens,
                  void* out, int B, int H, int d, int page_size, void* workspace,
                  unsigned int* err, int num_sms, cudaStream_t stream);

}  // namespace fa
