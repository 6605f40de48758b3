// fwd_sm100.cu -- fused attention forward pass for sm_100a.
//
// The method: the page "Flash Attention 是什么：2026 最新原理、架构演进与实战详解"
// (ai.lansai.wang), section 核心工作机制 -- Q, K and V are cut into blocks that
// fit on chip; each query block walks the key/value blocks, computes its
// scores, keeps a running row max m and normaliser l (the two update equations
// of section 关键术语解析, item 4, 在线 Softmax), corrects the partial output
// when m grows, and only the final O (plus the per-row log-sum-exp) is
// written to device memory.  The final division by l happens once, after the
// last block (page at zwxr.cn, section 3.1).
//
// B200 mapping (not the pages' design, which targets older GPUs):
//   * one CTA per 128-row query tile; K/V tiles of 128 keys stream through a
//     2-stage shared-memory ring filled by TMA (128-byte swizzle);
//   * the two products run on the 5th-generation tensor cores: S = Q K^T
//     (both operands in shared memory) and O += P V (P read from tensor
//     memory), with S, P and the O accumulator held in TMEM;
//   * warp roles: warps 0-3 do the softmax (one thread per query row, scores
//     read with tcgen05.ld), the O correction and the epilogue; warp 4 issues
//     TMA loads; warp 5 allocates TMEM and issues the MMAs;
//   * exp is evaluated as exp2 with scale*log2(e) folded into the scores.
//
// TMEM columns: S double buffer [0,128) and [128,256), O [256, 256+D),
// P (bf16 pairs) [384, 448).
#include <cuda_bf16.h>

#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int BM = 128;      // query rows per tile (MMA M)
constexpr int BN = 128;      // keys per K/V tile (MMA N of Q K^T, K of P V)
constexpr int kStages = 2;   // K/V ring depth
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr int kBoxBytes = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16

template <int D>
struct alignas(1024) FwdSmem {
    uint8_t q[BM * D * 2];
    uint8_t k[kStages][BN * D * 2];
    uint8_t v[kStages][BN * D * 2];
    uint64_t bar_q;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], s_free[2];
    uint64_t p_full, pv_done, drain;
    uint32_t tmem_base;
    int abort;
};

// All lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned int* err,
                                          volatile int* abort) {
    bool ok = mbar_wait(bar, parity, err, FA_DEVERR_TIMEOUT, abort);
    return __all_sync(0xffffffffu, ok);
}

template <int D, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const FwdParams p) {
    // ---- the work unit: (sequence/head, query tile) --------------------------
    int len, seq_start = 0, bh = 0, h = 0;
    if constexpr (VARLEN) {
        const int b = blockIdx.z;
        h = blockIdx.y;
        int s0 = p.cu_seqlens[b], s1 = p.cu_seqlens[b + 1];
        // keep every access inside the [total, H, d] tensors whatever the offsets say
        const int c0 = min(max(s0, 0), p.total), c1 = min(max(s1, c0), p.total);
        const int c1m = min(c1, c0 + p.N);
        if ((c0 != s0 || c1m != s1) && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
            record_error(p.err, FA_DEVERR_BAD_INPUT);
        seq_start = c0;
        len = c1m - c0;
    } else {
        bh = blockIdx.y;
        len = p.N;
    }
    const int nq = (len + BM - 1) / BM;
    // causal tiles near the end of the sequence carry the most work: start them first
    const int t = p.causal ? (nq - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
    if (t < 0 || t >= nq) return;
    const int nkv_all = (len + BN - 1) / BN;
    const int n_kv = p.causal ? min(t + 1, nkv_all) : nkv_all;

    extern __shared__ uint8_t smem_raw[];
    FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const uint32_t warp = warp_id_uniform();
    const uint32_t lane = lane_id();
    unsigned int* err = p.err;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        mbar_init(&sm.bar_q, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.s_full[s], 1);
            mbar_init(&sm.s_free[s], BM);
        }
        mbar_init(&sm.p_full, BM);
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int q_row0 = t * BM;

    if (warp == 4) {
        // ================= TMA producer =================
        if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row) {
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    if constexpr (VARLEN)
                        tma_load_3d(dst + cb * kBoxBytes, map, bar, cb * 64, h, seq_start + row);
                    else
                        tma_load_3d(dst + cb * kBoxBytes, map, bar, cb * 64, row, bh);
                }
            };
            mbar_arrive_expect_tx(&sm.bar_q, BM * D * 2);
            load_tile(sm.q, &tq, &sm.bar_q, q_row0);
            int issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                if (!mbar_wait(&sm.k_empty[st], ph ^ 1, err, FA_DEVERR_TIMEOUT, abort)) break;
                mbar_arrive_expect_tx(&sm.k_full[st], BN * D * 2);
                load_tile(sm.k[st], &tk, &sm.k_full[st], j * BN);
                if (!mbar_wait(&sm.v_empty[st], ph ^ 1, err, FA_DEVERR_TIMEOUT, abort)) {
                    issued = j;  // K of tile j is in flight, V is not
                    mbar_wait(&sm.k_full[st], ph, err, FA_DEVERR_TIMEOUT, nullptr);
                    break;
                }
                mbar_arrive_expect_tx(&sm.v_full[st], BN * D * 2);
                load_tile(sm.v[st], &tv, &sm.v_full[st], j * BN);
                issued = j + 1;
            }
            // Before the CTA may exit, every copy it started must have landed.
            // On the normal path the MMA warp has consumed them all already.
            mbar_wait(&sm.bar_q, 0, err, FA_DEVERR_TIMEOUT, nullptr);
            for (int j = max(0, issued - kStages); j < issued; ++j) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                mbar_wait(&sm.k_full[st], ph, err, FA_DEVERR_TIMEOUT, nullptr);
                mbar_wait(&sm.v_full[st], ph, err, FA_DEVERR_TIMEOUT, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);
            const uint32_t q_base = smem_u32(sm.q);
            auto issue_s = [&](int j) -> bool {
                const int st = j % kStages;
                const int sb = j & 1;
                if (!mbar_wait(&sm.k_full[st], (j / kStages) & 1, err, FA_DEVERR_TIMEOUT, abort))
                    return false;
                if (!mbar_wait(&sm.s_free[sb], ((j >> 1) & 1) ^ 1, err, FA_DEVERR_TIMEOUT, abort))
                    return false;
                tc_fence_after();
                const uint32_t k_base = smem_u32(sm.k[st]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    const uint64_t da = smem_desc_sw128(q_base + off, 16, 1024);
                    const uint64_t db = smem_desc_sw128(k_base + off, 16, 1024);
                    mma_ss(tmem + kColS + sb * BN, da, db, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&sm.s_full[sb]);
                tc_commit(&sm.k_empty[st]);
                return true;
            };
            bool ok = mbar_wait(&sm.bar_q, 0, err, FA_DEVERR_TIMEOUT, abort);
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + 1 < n_kv && !issue_s(j + 1)) break;
                const int st = j % kStages;
                if (!mbar_wait(&sm.p_full, j & 1, err, FA_DEVERR_TIMEOUT, abort)) break;
                if (!mbar_wait(&sm.v_full[st], (j / kStages) & 1, err, FA_DEVERR_TIMEOUT, abort))
                    break;
                tc_fence_after();
                const uint32_t v_base = smem_u32(sm.v[st]);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // 16 keys = 16 rows of 128 bytes in each 64-column block
                    const uint64_t db = smem_desc_sw128(v_base + kk * 16 * 128, kBoxBytes, 1024);
                    mma_ts(tmem + kColO, tmem + kColP + kk * 8, db, idesc_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&sm.pv_done);
                tc_commit(&sm.v_empty[st]);
            }
            // every MMA this thread issued must be complete before TMEM is freed
            tc_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, err, FA_DEVERR_TIMEOUT, nullptr);
        }
        __syncwarp();
    } else {
        // ================= softmax / correction / epilogue (warps 0-3) =================
        const int r = threadIdx.x;  // query row within the tile == TMEM lane
        const uint32_t lane_off = (warp * 32u) << 16;
        const int qrow = q_row0 + r;
        const float sl = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int sb = j & 1;
            if (!warp_wait(&sm.s_full[sb], (j >> 1) & 1, err, abort)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld32(tmem + lane_off + kColS + sb * BN + c * 32,
                          *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.s_free[sb]);

            // scaled scores in the log2 domain, masked entries -> -inf
            float x[BN];
            int limit = len - j * BN;                        // keys past the sequence end
            if (p.causal) limit = min(limit, qrow - j * BN + 1);  // keys after this row
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                const float s = __uint_as_float(sr[c]) * sl;
                x[c] = (c < limit) ? s : -INFINITY;
            }
            float mt = x[0];
#pragma unroll
            for (int c = 1; c < BN; ++c) mt = fmaxf(mt, x[c]);
            const float m_new = fmaxf(m, mt);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = ex2_approx(m - m_use);  // m = -inf -> 0

            if (j > 0) {
                // O and the P buffer are free once P V of the previous tile is done
                if (!warp_wait(&sm.pv_done, (j - 1) & 1, err, abort)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t orr[32];
                        tmem_ld32(tmem + lane_off + kColO + c * 32, orr);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
                        tmem_st32(tmem + lane_off + kColO + c * 32, orr);
                    }
                }
            }
            float rs = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                const float p0 = ex2_approx(x[c] - m_use);
                const float p1 = ex2_approx(x[c + 1] - m_use);
                rs += p0 + p1;
                pk[c / 2] = pack_bf16x2(p0, p1);
            }
            l = l * alpha + rs;
            m = m_new;
            tmem_st32(tmem + lane_off + kColP, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + kColP + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.p_full);
        }
        if (ok && warp_wait(&sm.pv_done, (n_kv - 1) & 1, err, abort)) {
            tc_fence_after();
            const bool store = qrow < len;
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow;
            if constexpr (VARLEN)
                orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                       (static_cast<int64_t>(seq_start + qrow) * p.H + h) * D;
            else
                orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                       (static_cast<int64_t>(bh) * p.N + qrow) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t orr[32];
                tmem_ld32(tmem + lane_off + kColO + c * 32, orr);
                tmem_wait_ld();
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(orr[e * 8 + 0]) * inv_l,
                                          __uint_as_float(orr[e * 8 + 1]) * inv_l);
                        w.y = pack_bf16x2(__uint_as_float(orr[e * 8 + 2]) * inv_l,
                                          __uint_as_float(orr[e * 8 + 3]) * inv_l);
                        w.z = pack_bf16x2(__uint_as_float(orr[e * 8 + 4]) * inv_l,
                                          __uint_as_float(orr[e * 8 + 5]) * inv_l);
                        w.w = pack_bf16x2(__uint_as_float(orr[e * 8 + 6]) * inv_l,
                                          __uint_as_float(orr[e * 8 + 7]) * inv_l);
                        dst[e] = w;
                    }
                }
            }
            if (store) {
                // lse = ln(sum exp(s)) = (m + log2 l) * ln 2 in the log2 domain used above
                const float lse = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
                if constexpr (VARLEN)
                    p.lse[static_cast<int64_t>(h) * p.total + seq_start + qrow] = lse;
                else
                    p.lse[static_cast<int64_t>(bh) * p.N + qrow] = lse;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

template <int D, bool VARLEN>
int launch_impl(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, cudaStream_t stream) {
    // Every CTA allocates all 512 TMEM columns, so one CTA per SM: ask for
    // enough shared memory that a second CTA cannot be co-resident.
    const size_t smem = sizeof(FwdSmem<D>) + 1024 > 120 * 1024 ? sizeof(FwdSmem<D>) + 1024
                                                               : 120 * 1024;
    auto kern = fa_fwd_kernel<D, VARLEN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FA_ERR_CUDA;
    dim3 grid;
    const int tiles = (p.N + BM - 1) / BM;
    if constexpr (VARLEN)
        grid = dim3(tiles, p.H, p.B);
    else
        grid = dim3(tiles, p.B * p.H, 1);
    kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

int launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, int d, bool varlen, cudaStream_t stream) {
    if (d == 128)
        return varlen ? launch_impl<128, true>(p, tq, tk, tv, stream)
                      : launch_impl<128, false>(p, tq, tk, tv, stream);
    if (d == 64)
        return varlen ? launch_impl<64, true>(p, tq, tk, tv, stream)
                      : launch_impl<64, false>(p, tq, tk, tv, stream);
    return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
