// bwd_sm100.cu -- attention backward pass for sm_100a.
//
// The page "Flash Attention 是什么：2026 最新原理、架构演进与实战详解"
// (ai.lansai.wang), section 核心工作机制, recomputation paragraph: the forward
// pass keeps each row's softmax statistics so that the backward pass can
// rebuild the probabilities tile by tile instead of storing the N x N matrix.
// With the saved log-sum-exp L_i the gradients of O = softmax(scale Q K^T) V
// for an output gradient dO are
//   P   = exp(scale Q K^T - L)          (rebuilt per tile)
//   dV  = P^T dO
//   dP  = dO V^T,   D_i = sum_c dO_ic O_ic
//   dS  = P o (dP - D)
//   dQ  = scale dS K,   dK = scale dS^T Q.
//
// B200 mapping (written for this part, not taken from the pages): one CTA per
// (sequence/head, 128-key block) keeps its K and V tiles in shared memory and
// the dK, dV accumulators in tensor memory, and streams the query tiles that
// see its keys (all of them, or those on and below the diagonal when causal).
// Per query tile, five tcgen05 MMAs:
//   S^T  = K Q_i^T          (TMEM, lanes = keys)
//   dV  += P^T dO_i         (P^T from TMEM as bf16)
//   dP^T = V dO_i^T         (TMEM)
//   dQ_i = dS K             (dS from shared memory, written over the dO_i
//                            tile once its last reader has completed)
//   dK  += dS^T Q_i         (the same shared-memory tile, read K-major)
// Warpgroup 0 (one thread per key) turns S^T into P^T and dP^T into dS^T;
// warpgroup 1 adds each dQ_i into an fp32 accumulator in device memory (the
// key blocks of a head all contribute to every dQ row) and writes dK, dV at
// the end; warp 8 issues the MMAs, warp 9 the TMA loads (warps 10, 11 only
// complete warpgroup 2, whose registers setmaxnreg moves to warpgroup 0).
// dP^T of a tile needs no P^T, so it is issued as soon as the previous dQ_i
// has left TMEM: warpgroup 0 finds it ready right after P^T, and the tensor
// pipe runs dV and the next S^T while warpgroup 0 forms dS.  A prep
// kernel forms D and the log2-domain statistics and clears the dQ
// accumulator; a final kernel rounds dQ to bf16.
//
// TMEM columns: S^T [0,128) (P^T as bf16 pairs in [0,64)), dP^T [128,256)
// (dQ_i reuses [128,128+D) once warpgroup 0 has read dP^T), dV [256,256+D),
// dK [384,384+D).
#include <cuda_bf16.h>

#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBT = 128;            // keys per CTA, queries per tile
constexpr int kBwdThreads = 384;    // 12 warps: 3 warpgroups
// setmaxnreg split of the 168 registers per thread the block launches with
// (65536 / 384, rounded down to 8): warpgroup 0 holds a whole S^T or dP^T row
// (128 values) next to its P^T row, warpgroup 1 a whole dQ_i row
constexpr uint32_t kRegsWg0 = 216, kRegsWg1 = 184, kRegsWg2 = 104;
static_assert(kRegsWg0 + kRegsWg1 + kRegsWg2 <= 3 * 168, "register split exceeds the launch share");
constexpr int kBwdHeadGroup = 4;    // (sequence, head) units scheduled together
constexpr int kBoxB = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

template <int D>
struct alignas(1024) BwdSmem {
    uint8_t k[kBT * D * 2];
    uint8_t v[kBT * D * 2];
    uint8_t q[2][kBT * D * 2];
    // dO_i (128 x D), then dS_i (128 x 128) once dO_i is consumed
    uint8_t dout[2][kBT * kBT * 2];
    // one 128-row x 32-column fp32 slice of dQ_i on its way to the
    // accumulator (128-byte swizzle, as the reduce's tensor map reads it)
    float dq_stage[kBT * 32];
    float nlse2[2][kBT];           // -(log2-domain statistics) of the tile's rows
    float ndsum[2][kBT];           // -D of the tile's rows
    uint64_t kv_full;
    uint64_t in_full[2], in_free[2];  // Q/dO/statistics slot loaded / released
    uint64_t s_full, p_full, dp_full, dv_done, ds_full, dq_full, dq_free;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct BwdParams {
    const float* lse2;   // per row of O: lse * log2(e)
    const float* dsum;   // per row of O: D
    float* dq_acc;       // [B*H*N*D] fp32, cleared by the prep kernel
    void* dk;
    void* dv;
    int B, H, H_kv, N, causal;  // query head h uses K/V head h / (H / H_kv)
    const int32_t* cu_seqlens;  // packed sequences: offsets [B+1]; N is the longest length
    int total;                  // packed sequences: rows of q, k, v
    float scale, scale_log2;
    unsigned int* err;
};

__device__ __forceinline__ bool bwd_warp_wait(uint64_t* bar, uint32_t parity, unsigned int* err,
                                              volatile int* abort) {
    bool ok = mbar_wait(bar, parity, err, FA_DEVERR_TIMEOUT, abort);
    return __all_sync(0xffffffffu, ok);
}

// 32 TMEM columns of bf16 pairs (64 values) <- 64 fp32 values
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}

// ---------------------------------------------------------------------------
// prep: D_i = dO_i . O_i, lse2_i = lse_i * log2(e), dQ accumulator rows = 0.
// One warp per row r of O.  lse_total = 0: lse, the statistics and the
// accumulator are indexed like the rows of O; otherwise O is packed
// [total, H, d] (row r = token r / H, head r % H) and lse, the statistics and
// the accumulator rows are head-major ([H, total], [H, total, d]), so that a
// tile's rows are contiguous in them.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                       const float* __restrict__ lse, float* __restrict__ lse2,
                       float* __restrict__ dsum, float* __restrict__ dq_acc, int64_t rows, int H,
                       int64_t lse_total) {
    constexpr int PER = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31;
    for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
         r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
        const __nv_bfloat16* orow = o + r * D + lane * PER;
        const __nv_bfloat16* grow = dout + r * D + lane * PER;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < PER; e += 2) {
            const uint32_t wo = *reinterpret_cast<const uint32_t*>(orow + e);
            const uint32_t wg = *reinterpret_cast<const uint32_t*>(grow + e);
            float o0, o1, g0, g1;
            unpack_bf16x2(wo, o0, o1);
            unpack_bf16x2(wg, g0, g1);
            acc = fmaf(o0, g0, fmaf(o1, g1, acc));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const int64_t li = lse_total ? (r % H) * lse_total + r / H : r;
        if (lane == 0) {
            dsum[li] = acc;
            lse2[li] = lse[li] * 1.4426950408889634f;
        }
        float4* dq = reinterpret_cast<float4*>(dq_acc + li * D);
        for (int c = lane; c < D / 4; c += 32) dq[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// dq (bf16) <- dQ accumulator (fp32), 8 values per thread; with lse_total
// the accumulator is head-major [H, total, D] and dq packed [total, H, D]
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_dq_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq,
                     int64_t n8, int H, int64_t lse_total) {
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < n8;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t src = x;  // in units of 8 values
        if (lse_total) {
            const int64_t r = x / (D / 8), c = x - r * (D / 8);  // row of dq, 8-column chunk
            src = ((r % H) * lse_total + r / H) * (D / 8) + c;
        }
        const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * src];
        const float4 b = reinterpret_cast<const float4*>(dq_acc)[2 * src + 1];
        uint4 w;
        w.x = pack_bf16x2(a.x, a.y);
        w.y = pack_bf16x2(a.z, a.w);
        w.z = pack_bf16x2(b.x, b.y);
        w.w = pack_bf16x2(b.z, b.w);
        reinterpret_cast<uint4*>(dq)[x] = w;
    }
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------
// VARLEN: q, k, v, o, dout packed [total, heads, d] (maps over (d, heads,
// total), 64 x 1 x 128 boxes; the statistics and the fp32 dQ accumulator are
// head-major, [H, total] and [H, total, d]); sequence b owns rows cu_seqlens[b] ..
// cu_seqlens[b+1]-1 and attends within itself.  Rows of a tile past its
// sequence belong to the next one (or lie past the tensor): their P is 0
// (statistics lse = +inf), so their dQ rows add exact zeros and their keys
// contribute nothing; dK, dV rows past the sequence are not stored.
template <int D, bool VARLEN>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                  const __grid_constant__ CUtensorMap tdq, const BwdParams p) {
    // ---- work unit: (sequence/head, 128-key block), longest first within
    // groups of kBwdHeadGroup heads (under a causal mask key block 0 meets
    // every query tile)
    const int units = p.B * p.H_kv;  // (sequence, K/V head)
    const int nkb = (p.N + kBT - 1) / kBT;
    const int gidx = static_cast<int>(blockIdx.x) / (kBwdHeadGroup * nkb);
    const int ug = min(kBwdHeadGroup, units - gidx * kBwdHeadGroup);
    const int within = static_cast<int>(blockIdx.x) - gidx * kBwdHeadGroup * nkb;
    const int jb = within / ug;
    const int bh = gidx * kBwdHeadGroup + (within - jb * ug);  // flat (sequence, K/V head)
    if (jb >= nkb || bh >= units) return;
    // the sequence: its first packed row and length (fixed length: N rows)
    int seq0 = 0, len = p.N;
    if constexpr (VARLEN) {
        const int b = bh / p.H_kv;
        const int s0 = p.cu_seqlens[b], s1 = p.cu_seqlens[b + 1];
        // keep every access inside the packed tensors whatever the offsets say
        const int c0 = min(max(s0, 0), p.total), c1 = min(max(s1, c0), p.total);
        const int c1m = min(c1, c0 + p.N);
        if ((c0 != s0 || c1m != s1) && jb == 0 && bh % p.H_kv == 0 && threadIdx.x == 0)
            record_error(p.err, FA_DEVERR_BAD_INPUT);
        seq0 = c0;
        len = c1m - c0;
    }
    const int nkb_seq = (len + kBT - 1) / kBT;
    if (jb >= nkb_seq) return;
    const int key0 = jb * kBT;
    const int i_first = p.causal ? jb : 0;
    const int nt = nkb_seq - i_first;  // query tiles of one query head that see this key block
    // the CTA walks the query tiles of every query head of its K/V head's
    // group (dK, dV sum over all of them): tile t is query tile
    // i_first + t % nt of query head t / nt of the group
    const int G = p.H / p.H_kv;
    const int ntt = G * nt;
    const int qh0 = (bh / p.H_kv) * p.H + (bh % p.H_kv) * G;  // flat first query head
    auto tile_q0 = [&](int t) { return (i_first + t % nt) * kBT; };
    auto tile_qh = [&](int t) { return qh0 + t / nt; };
    // row `row` of the sequence for (flat) head `head` as tensor-map
    // coordinates, and the index of that row of O (statistics)
    auto map_row = [&](int row) { return VARLEN ? seq0 + row : row; };
    auto map_head = [&](int head, int heads) { return VARLEN ? head % heads : head; };
    auto stat_index = [&](int head, int row) -> int64_t {
        return VARLEN ? static_cast<int64_t>(head % p.H) * p.total + seq0 + row
                      : static_cast<int64_t>(head) * p.N + row;
    };

    extern __shared__ uint8_t bwd_smem_raw[];
    BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(
        (reinterpret_cast<uintptr_t>(bwd_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t warp = warp_id_uniform();
    const uint32_t lane = lane_id();
    unsigned int* err = p.err;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        mbar_init(&sm.kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.in_full[s], 1 + 32);  // TMA bytes + the producer lanes' statistics
            mbar_init(&sm.in_free[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, kBT);
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.dv_done, 1);
        mbar_init(&sm.ds_full, kBT);
        mbar_init(&sm.dq_full, 1);
        mbar_init(&sm.dq_free, kBT);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp >= 8) regs_dec<kRegsWg2>();
    if (warp == 9) {
        // ================= TMA producer (+ per-tile statistics) =================
        // fixed length: maps over (d, N, sequences * heads); packed: (d, heads, total)
        auto load2 = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row, int head,
                         int heads) {
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
                if constexpr (VARLEN)
                    tma_load_3d(dst + cb * kBoxB, map, bar, cb * 64, map_head(head, heads),
                                map_row(row));
                else
                    tma_load_3d(dst + cb * kBoxB, map, bar, cb * 64, row, head);
            }
        };
        bool ok = true;
        if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            tma_prefetch_desc(&tdo);
            mbar_arrive_expect_tx(&sm.kv_full, 2 * kBT * D * 2);
            load2(sm.k, &tk, &sm.kv_full, key0, bh, p.H_kv);
            load2(sm.v, &tv, &sm.kv_full, key0, bh, p.H_kv);
        }
        int issued = 0;
        for (int t = 0; t < ntt; ++t) {
            const int s = t & 1;
            if (t >= 2 && !bwd_warp_wait(&sm.in_free[s], ((t - 2) >> 1) & 1, err, abort)) {
                ok = false;
                break;
            }
            const int q0 = tile_q0(t), qh = tile_qh(t);
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.in_full[s], 2 * kBT * D * 2);
                load2(sm.q[s], &tq, &sm.in_full[s], q0, qh, p.H);
                load2(sm.dout[s], &tdo, &sm.in_full[s], q0, qh, p.H);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = lane * 4 + e, qr = q0 + r;
                const bool in = qr < len;
                const int64_t gi = in ? stat_index(qh, qr) : 0;
                sm.nlse2[s][r] = in ? -p.lse2[gi] : -INFINITY;  // rows past N: P = 0
                sm.ndsum[s][r] = in ? -p.dsum[gi] : 0.f;
            }
            mbar_arrive(&sm.in_full[s]);
            issued = t + 1;
        }
        // every copy this CTA started must land before it exits
        if (lane == 0) {
            mbar_wait(&sm.kv_full, 0, err, FA_DEVERR_TIMEOUT, nullptr);
            for (int t = max(0, issued - 2); t < issued; ++t)
                mbar_wait(&sm.in_full[t & 1], (t >> 1) & 1, err, FA_DEVERR_TIMEOUT, nullptr);
        }
        (void)ok;
        __syncwarp();
    } else if (warp == 8) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_kk = idesc_bf16_f32(kBT, kBT, 0, 0);   // S^T, dP^T
            constexpr uint32_t idesc_tm = idesc_bf16_f32(kBT, D, 0, 1);     // dV, dK
            constexpr uint32_t idesc_mm = idesc_bf16_f32(kBT, D, 1, 1);     // dQ
            constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
            constexpr uint32_t kLboK = (16u >> 4) << 16;
            constexpr uint32_t kLboMN = (static_cast<uint32_t>(kBoxB) >> 4) << 16;
            auto lo = [](const void* ptr) { return smem_u32(ptr) >> 4; };
            auto dk_ = [&](uint32_t base_lo, uint32_t off) {  // K-major operand
                return (static_cast<uint64_t>(kDescHi) << 32) | (kLboK | (base_lo + off));
            };
            auto dmn = [&](uint32_t base_lo, uint32_t off) {  // MN-major operand
                return (static_cast<uint64_t>(kDescHi) << 32) | (kLboMN | (base_lo + off));
            };
            // D[col] (+)= A (rows of a, K-major) * B (rows of b, K-major)^T over d
            auto issue_kk = [&](uint32_t col, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t o = (kk >> 2) * (kBoxB >> 4) + (kk & 3) * 2;
                    mma_ss(tmem + col, dk_(a_lo, o), dk_(b_lo, o), idesc_kk, kk > 0 ? 1u : 0u);
                }
            };
            // D[col] (+)= A (bf16 pairs in TMEM at acol) * B (MN-major rows) over 128
            auto issue_tm = [&](uint32_t col, uint32_t acol, uint32_t b_lo, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kBT / 16; ++kk)
                    mma_ts(tmem + col, tmem + acol + kk * 8, dmn(b_lo, kk * 128), idesc_tm,
                           (acc || kk > 0) ? 1u : 0u);
            };
            // D[col] (+)= A (K-major rows of a) * B (MN-major rows) over 128
            auto issue_sm = [&](uint32_t col, uint32_t a_lo, uint32_t b_lo, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kBT / 16; ++kk)
                    mma_ss(tmem + col, dk_(a_lo, (kk >> 2) * (kBoxB >> 4) + (kk & 3) * 2),
                           dmn(b_lo, kk * 128), idesc_tm, (acc || kk > 0) ? 1u : 0u);
            };
            // D[col] = A (MN-major) * B (MN-major) over 128
            auto issue_mm = [&](uint32_t col, uint32_t a_lo, uint32_t b_lo) {
#pragma unroll
                for (int kk = 0; kk < kBT / 16; ++kk)
                    mma_ss(tmem + col, dmn(a_lo, kk * 128), dmn(b_lo, kk * 128), idesc_mm,
                           kk > 0 ? 1u : 0u);
            };
            const uint32_t k_lo = lo(sm.k), v_lo = lo(sm.v);
            // Per tile: dV once P^T is in TMEM, then the next tile's S^T, dQ_i
            // and dK once dS is in shared memory, then the next tile's dP^T
            // once dQ_i has been read out of the columns it shares;
            // warpgroup 0 forms dS while dV and the next S^T run
            bool ok = mbar_wait(&sm.kv_full, 0, err, FA_DEVERR_TIMEOUT, abort) &&
                      mbar_wait(&sm.in_full[0], 0, err, FA_DEVERR_TIMEOUT, abort);
            if (ok) {
                tc_fence_after();
                issue_kk(kColS, k_lo, lo(sm.q[0]));  // S^T = K Q_0^T
                tc_commit(&sm.s_full);
                issue_kk(kColDP, v_lo, lo(sm.dout[0]));  // dP^T = V dO_0^T
                tc_commit(&sm.dp_full);
            }
            for (int t = 0; ok && t < ntt; ++t) {
                const int s = t & 1;
                const uint32_t ph = t & 1;
                const uint32_t q_lo = lo(sm.q[s]), do_lo = lo(sm.dout[s]);
                if (!mbar_wait(&sm.p_full, ph, err, FA_DEVERR_TIMEOUT, abort)) break;
                tc_fence_after();
                issue_tm(kColDV, kColS, do_lo, t > 0);  // dV += P^T dO_i
                tc_commit(&sm.dv_done);                 // dO_i's last reader before dS
                const int s1 = (t + 1) & 1;
                if (t + 1 < ntt) {
                    // S^T of the next tile (its columns held P^T, read by dV above)
                    if (!mbar_wait(&sm.in_full[s1], ((t + 1) >> 1) & 1, err, FA_DEVERR_TIMEOUT,
                                   abort))
                        break;
                    tc_fence_after();
                    issue_kk(kColS, k_lo, lo(sm.q[s1]));
                    tc_commit(&sm.s_full);
                }
                if (!mbar_wait(&sm.ds_full, ph, err, FA_DEVERR_TIMEOUT, abort)) break;
                tc_fence_after();
                issue_mm(kColDP, do_lo, k_lo);  // dQ_i = dS K (dS in the dO_i slot)
                tc_commit(&sm.dq_full);
                issue_sm(kColDK, do_lo, q_lo, t > 0);  // dK += dS^T Q_i, same tile K-major
                tc_commit(&sm.in_free[s]);
                if (t + 1 < ntt) {
                    // dP^T of the next tile, once dQ_i has left its columns
                    if (!mbar_wait(&sm.dq_free, ph, err, FA_DEVERR_TIMEOUT, abort)) break;
                    tc_fence_after();
                    issue_kk(kColDP, v_lo, lo(sm.dout[s1]));
                    tc_commit(&sm.dp_full);
                }
            }
            // every MMA issued must be complete before TMEM is freed
            tc_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, err, FA_DEVERR_TIMEOUT, nullptr);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ================= warpgroup 0: P^T and dS^T, one thread per key =================
        regs_inc<kRegsWg0>();
        const int r = threadIdx.x;  // TMEM lane == key row of the block
        const uint32_t lane_off = ((warp & 3) * 32u) << 16;
        const int key = key0 + r;
        const bool key_in = key < len;
        const float sl = p.scale_log2;
        for (int t = 0; t < ntt; ++t) {
            const int s = t & 1;
            const uint32_t ph = t & 1;
            const int q0 = tile_q0(t);
            const bool diag = p.causal && (i_first + t % nt == jb);
            if (!bwd_warp_wait(&sm.s_full, ph, err, abort)) break;
            tc_fence_after();
            // P^T = 2^(scale log2e S^T - lse2); keys past N, queries past N
            // (lse2 = +inf) and, on the diagonal, keys after the query give 0
            uint32_t pk[kBT / 2];
            {
                uint32_t x[kBT];  // the whole S^T row, one wait for all four loads
#pragma unroll
                for (int c = 0; c < kBT / 32; ++c)
                    tmem_ld32(tmem + lane_off + kColS + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&x[c * 32]));
                tmem_wait_ld();
                const float4* l4 = reinterpret_cast<const float4*>(sm.nlse2[s]);
                const uint64_t sl2 = f2_pack(sl, sl);
                if (key_in && !diag) {
#pragma unroll
                    for (int e4 = 0; e4 < kBT / 4; ++e4) {
                        const float4 lv = l4[e4];
                        const uint64_t a = f2_fma(f2_pack(__uint_as_float(x[4 * e4]),
                                                          __uint_as_float(x[4 * e4 + 1])),
                                                  sl2, f2_pack(lv.x, lv.y));
                        const uint64_t b = f2_fma(f2_pack(__uint_as_float(x[4 * e4 + 2]),
                                                          __uint_as_float(x[4 * e4 + 3])),
                                                  sl2, f2_pack(lv.z, lv.w));
                        pk[e4 * 2] = pack_bf16x2(ex2_approx(f2_lo(a)), ex2_approx(f2_hi(a)));
                        pk[e4 * 2 + 1] = pack_bf16x2(ex2_approx(f2_lo(b)), ex2_approx(f2_hi(b)));
                    }
                } else {
#pragma unroll
                    for (int e4 = 0; e4 < kBT / 4; ++e4) {
                        const float4 lv = l4[e4];
                        const float ls[4] = {lv.x, lv.y, lv.z, lv.w};
                        float pv[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int e = e4 * 4 + u;
                            float v = ex2_approx(fmaf(__uint_as_float(x[e]), sl, ls[u]));
                            if (!key_in || (diag && key > q0 + e)) v = 0.f;
                            pv[u] = v;
                        }
                        pk[e4 * 2] = pack_bf16x2(pv[0], pv[1]);
                        pk[e4 * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                    }
                }
            }
            tmem_st32(tmem + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full);
            // dS^T = P^T o (dP^T - D), packed over pk; written transposed
            // (row = key) into the dO_i slot once dV, the slot's last reader
            // (dP^T has completed), is done: dQ_i reads it as dS (MN-major),
            // dK as dS^T (K-major)
            if (!bwd_warp_wait(&sm.dp_full, ph, err, abort)) break;
            tc_fence_after();
            {
                uint32_t y[kBT];
#pragma unroll
                for (int c = 0; c < kBT / 32; ++c)
                    tmem_ld32(tmem + lane_off + kColDP + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&y[c * 32]));
                tmem_wait_ld();
                const float4* d4 = reinterpret_cast<const float4*>(sm.ndsum[s]);
#pragma unroll
                for (int e4 = 0; e4 < kBT / 4; ++e4) {
                    const float4 dv4 = d4[e4];
                    const int e = e4 * 4;
                    const uint32_t w0 = pk[e4 * 2], w1 = pk[e4 * 2 + 1];
                    const uint64_t a = f2_mul(f2_add(f2_pack(__uint_as_float(y[e]),
                                                             __uint_as_float(y[e + 1])),
                                                     f2_pack(dv4.x, dv4.y)),
                                              f2_pack(__uint_as_float(w0 << 16),
                                                      __uint_as_float(w0 & 0xffff0000u)));
                    const uint64_t b = f2_mul(f2_add(f2_pack(__uint_as_float(y[e + 2]),
                                                             __uint_as_float(y[e + 3])),
                                                     f2_pack(dv4.z, dv4.w)),
                                              f2_pack(__uint_as_float(w1 << 16),
                                                      __uint_as_float(w1 & 0xffff0000u)));
                    pk[e4 * 2] = pack_bf16x2(f2_lo(a), f2_hi(a));
                    pk[e4 * 2 + 1] = pack_bf16x2(f2_lo(b), f2_hi(b));
                }
            }
            // every thread has read its dP^T row: dQ_i may overwrite it once
            // ds_full completes
            if (!bwd_warp_wait(&sm.dv_done, ph, err, abort)) break;
            // row r of the dS tile: queries [32c, 32c+32) are box c/2, 16-byte
            // chunks (c%2)*4 .. +3 of the 128-byte row, 128-byte swizzle
            uint8_t* ds_tile = sm.dout[s];
#pragma unroll
            for (int c = 0; c < kBT / 32; ++c) {
                uint8_t* row = ds_tile + (c >> 1) * kBoxB + r * 128;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int chunk = (c & 1) * 4 + h;
                    const uint32_t* w = &pk[c * 16 + h * 4];
                    *reinterpret_cast<uint4*>(row + ((chunk ^ (r & 7)) * 16)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(&sm.ds_full);
        }
    } else if (warp < 8) {
        // ================= warpgroup 1: dQ_i accumulation, then dK and dV =================
        regs_inc<kRegsWg1>();
        const int r = threadIdx.x - 128;
        const uint32_t lane_off = ((warp & 3) * 32u) << 16;
        bool ok = true;
        for (int t = 0; t < ntt; ++t) {
            // the four warps leave together (they share named barriers below)
            if (!bar_and_named(2, kBT, mbar_wait(&sm.dq_full, t & 1, err, FA_DEVERR_TIMEOUT,
                                                 abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // dQ_i (TMEM lane == query row) in slices of 32 columns: each row
            // to the swizzled staging tile, then one TMA reduce-add of the
            // 128 x 32 slice into the accumulator (rows past N are clipped)
            const int q0 = tile_q0(t), qh = tile_qh(t);
            uint8_t* stage = reinterpret_cast<uint8_t*>(sm.dq_stage);
            // all of dQ_i into registers first, so that its TMEM columns are
            // released to the next dP^T before the reductions
            uint32_t z[D / 32][32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_off + kColDP + c * 32, z[c]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.dq_free);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                bar_sync_named(1, kBT);  // the previous slice's reduce has read the tile
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(stage + r * 128 + ((j ^ (r & 7)) * 16)) =
                        make_float4(__uint_as_float(z[c][4 * j]) * p.scale,
                                    __uint_as_float(z[c][4 * j + 1]) * p.scale,
                                    __uint_as_float(z[c][4 * j + 2]) * p.scale,
                                    __uint_as_float(z[c][4 * j + 3]) * p.scale);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                bar_sync_named(1, kBT);  // every row is in the tile
                if (r == 0) {
                    if constexpr (VARLEN)  // head-major accumulator (d, total, H)
                        tma_reduce_add_3d(&tdq, stage, c * 32, seq0 + q0, qh % p.H);
                    else
                        tma_reduce_add_3d(&tdq, stage, c * 32, q0, qh);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
            }
        }
        if (r == 0) bulk_wait_group0();  // the reductions have landed
        if (ok) {
            // every MMA has completed (the last dq_full follows the last one);
            // the whole warp loads (tcgen05.ld is warp-wide), rows past the
            // sequence are not stored
            const int key = key0 + r;
            const bool store = key < len;
            const int64_t krow = VARLEN ? static_cast<int64_t>(seq0 + key) * p.H_kv + bh % p.H_kv
                                        : static_cast<int64_t>(bh) * p.N + key;
            __nv_bfloat16* dvr = reinterpret_cast<__nv_bfloat16*>(p.dv) + krow * D;
            __nv_bfloat16* dkr = reinterpret_cast<__nv_bfloat16*>(p.dk) + krow * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = which ? kColDK : kColDV;
                const float mul = which ? p.scale : 1.f;
                __nv_bfloat16* out = which ? dkr : dvr;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t z[32];
                    tmem_ld32(tmem + lane_off + col + c * 32, z);
                    tmem_wait_ld();
                    if (store) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(z[e * 8]) * mul, __uint_as_float(z[e * 8 + 1]) * mul);
                            w.y = pack_bf16x2(__uint_as_float(z[e * 8 + 2]) * mul, __uint_as_float(z[e * 8 + 3]) * mul);
                            w.z = pack_bf16x2(__uint_as_float(z[e * 8 + 4]) * mul, __uint_as_float(z[e * 8 + 5]) * mul);
                            w.w = pack_bf16x2(__uint_as_float(z[e * 8 + 6]) * mul, __uint_as_float(z[e * 8 + 7]) * mul);
                            reinterpret_cast<uint4*>(out + c * 32)[e] = w;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 8) tmem_dealloc(tmem, 512);
}

template <int D>
int launch_bwd_impl(const void* o, const void* dout, const float* lse, float* lse2, float* dsum,
                    float* dq_acc, void* dq, const CUtensorMap& tq, const CUtensorMap& tk,
                    const CUtensorMap& tv, const CUtensorMap& tdo, const CUtensorMap& tdq,
                    const BwdParams& p, int num_sms, cudaStream_t stream) {
    const bool varlen = p.cu_seqlens != nullptr;
    const int64_t rows = varlen ? static_cast<int64_t>(p.total) * p.H
                                : static_cast<int64_t>(p.B) * p.H * p.N;
    fa_bwd_prep_kernel<D><<<num_sms * 8, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lse2,
        dsum, dq_acc, rows, p.H, varlen ? p.total : 0);
    const size_t smem = sizeof(BwdSmem<D>) + 1024;
    auto kern = varlen ? fa_bwd_kernel<D, true> : fa_bwd_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FA_ERR_CUDA;
    const long long ctas = static_cast<long long>((p.N + kBT - 1) / kBT) * p.B * p.H_kv;
    if (ctas > 0x7fffffffLL) return FA_ERR_SHAPE;
    kern<<<dim3(static_cast<unsigned>(ctas)), kBwdThreads, smem, stream>>>(tq, tk, tv, tdo, tdq,
                                                                           p);
    fa_bwd_dq_kernel<D><<<num_sms * 8, 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                          rows * D / 8, p.H,
                                                          varlen ? p.total : 0);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

size_t bwd_dq_acc_offset(int B, int H, int N) {
    const size_t rows = static_cast<size_t>(B) * H * N;
    return (2 * rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
}

size_t bwd_workspace_bytes(int B, int H, int N, int d) {
    return bwd_dq_acc_offset(B, H, N) + static_cast<size_t>(B) * H * N * d * sizeof(float);
}

int launch_bwd(const void* o, const void* dout, const float* lse, void* dq, void* dk, void* dv,
               const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& tdo, const CUtensorMap& tdq, int B, int H, int H_kv, int N, int d,
               int causal, float scale, void* workspace, unsigned int* err, int num_sms,
               cudaStream_t stream, const int32_t* cu_seqlens, int total) {
    // statistics and the dQ accumulator: one entry per row of O
    const int Bw = cu_seqlens ? 1 : B, Nw = cu_seqlens ? total : N;
    const size_t rows = static_cast<size_t>(Bw) * H * Nw;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* lse2 = reinterpret_cast<float*>(ws);
    float* dsum = lse2 + rows;
    float* dq_acc = reinterpret_cast<float*>(ws + bwd_dq_acc_offset(Bw, H, Nw));
    BwdParams p{};
    p.lse2 = lse2;
    p.dsum = dsum;
    p.dq_acc = dq_acc;
    p.dk = dk;
    p.dv = dv;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.N = N;
    p.causal = causal;
    p.cu_seqlens = cu_seqlens;
    p.total = total;
    p.scale = scale;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.err = err;
    if (d == 128)
        return launch_bwd_impl<128>(o, dout, lse, lse2, dsum, dq_acc, dq, tq, tk, tv, tdo, tdq,
                                    p, num_sms, stream);
    if (d == 64)
        return launch_bwd_impl<64>(o, dout, lse, lse2, dsum, dq_acc, dq, tq, tk, tv, tdo, tdq,
                                   p, num_sms, stream);
    return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
