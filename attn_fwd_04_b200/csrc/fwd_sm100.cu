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
//   * one CTA per 256-row query block, processed as two 128-row tiles that
//     share every K/V tile; K and V tiles of 128 keys stream through a 4-slot
//     shared-memory ring filled by TMA (128-byte swizzle);
//   * both products run on the 5th-generation tensor cores: S = Q K^T (both
//     operands in shared memory) and O += P V (P read from tensor memory);
//     S, P and both O accumulators live in TMEM (all 512 columns);
//   * warp roles (512 threads): warpgroups 0 and 1 run the softmax of tile 0
//     and tile 1 (one thread per query row), so one tile's softmax overlaps
//     the other tile's MMAs; each also rescales its own O accumulator when
//     the running max grows; warpgroup 2 writes the epilogue; in warpgroup 3,
//     warp 12 issues the MMAs and warp 13 the TMA loads.  Registers are moved
//     to the softmax warpgroups with setmaxnreg (kRegsSoftmax etc. below);
//   * exp is exp2 with scale*log2(e) folded in (the polynomial path below can
//     take a share of the exponentials off the special-function unit; it is
//     switched off because it measured slower here); O is rescaled only when
//     the running max has grown by more than 2^8 (the stale max is used for
//     both the numerator and l, so the result is unchanged up to rounding).
//   * opt-in (fa_fwd_set_cta_pairs, d = 128, fixed length): CTA pairs whose
//     products span both SMs (tcgen05 cta_group::2, M = 256), each CTA loading
//     half of every K/V tile; it moves half the K/V bytes per query row but
//     couples both CTAs' softmax to every product, and measured slower.
//
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [384,384+D).
// P_t (bf16 pairs) overwrites the first 64 columns of S_t; the next S_t is
// issued behind P_t V in the same in-order MMA stream.
#include <cuda_bf16.h>

#include <type_traits>

#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int BM = 128;       // query rows per tile (MMA M)
constexpr int BN = 128;       // keys per K/V tile
constexpr int kSlots = 4;     // K/V ring slots (each holds one K or one V tile)
constexpr int kThreads = 512;
// setmaxnreg shares (registers per thread) of the softmax warpgroups, the
// epilogue warpgroup and warpgroup 3 (TMA and MMA warps).  They come out of
// the 128 per thread the block launches with (65536 / 512): a split whose sum
// exceeded 4 x 128 would make the increase wait forever.
constexpr uint32_t kRegsSoftmax = 192, kRegsEpilogue = 72, kRegsIssue = 56;
static_assert(2 * kRegsSoftmax + kRegsEpilogue + kRegsIssue <= 4 * 128,
              "register split exceeds the launch share");
constexpr int kHeadGroup = 4;  // (sequence, head) units scheduled together
constexpr uint32_t kTmemCols = 512;
__host__ __device__ constexpr uint32_t col_s(int t) { return 128u * t; }        // S_t / P_t
__host__ __device__ constexpr uint32_t col_o(int t) { return 256u + 128u * t; }  // O_t
constexpr int kBoxBytes = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16
// P is computed against the running max of earlier steps; only when a row's
// sum of P exceeds 2^16 (so some score beat that max by more than 2^16 / 128)
// is the row's true max taken, O and l rescaled and P recomputed.
constexpr float kLazySum = 65536.f;
// Exponentials of pairs (c/2) % 8 in [0, kPolyPairs) are evaluated with the
// FMA-pipe polynomial below, the rest with the special-function unit.
constexpr int kPolyPairs = 0;
// 2^f on [-1/2, 1/2], degree-3 minimax in relative error (7.5e-5), fitted by
// the Remez exchange in exp2_poly_remez.py beside this file.
constexpr float kExp2P0 = 0.9999280571937561f, kExp2P1 = 0.6932609677314758f,
                kExp2P2 = 0.2426111251115799f, kExp2P3 = 0.0551716685295105f;

// PAIR: the CTA is one of a pair whose products run on both SMs' tensor cores
// (M = 256: each CTA's query tile is half of the A operand); a ring slot then
// holds this CTA's half of a K tile (64 keys) or of a V tile (64 of the 128
// dimensions), so the ring has twice the slots in the same space.
template <bool PAIR> constexpr int ring_slots() { return PAIR ? 2 * kSlots : kSlots; }

template <int D, bool PAIR>
struct alignas(1024) FwdSmem {
    static constexpr int kRing = ring_slots<PAIR>();
    static constexpr int kSlotBytes = PAIR ? BN * D : BN * D * 2;
    uint8_t q[2][BM * D * 2];
    uint8_t kv[kRing][kSlotBytes];
    float row_m[2][BM];   // final running max (log2 domain) per row
    float row_l[2][BM];   // final normaliser per row
    uint64_t q_full[2];
    uint64_t kv_full[kRing], kv_empty[kRing];
    uint64_t s_full[2], p_full[2], pv_done[2], stats_full[2];
    uint64_t vfix;   // paged: the last V tile's rows past the sequence are zeroed
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned int* err,
                                          volatile int* abort, uint64_t limit_ns) {
    bool ok = mbar_wait(bar, parity, err, FA_DEVERR_TIMEOUT, abort, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// K/V ring position of tile j's K (v = 0) or V (v = 1) in a ring of R slots
template <int R = kSlots>
__device__ __forceinline__ int ring_slot(int j, int v) { return (2 * j + v) % R; }
template <int R = kSlots>
__device__ __forceinline__ uint32_t ring_phase(int j, int v) { return ((2 * j + v) / R) & 1; }

// Max (or, for a negative scale, min) of the 128 raw scores of a row.
__device__ __forceinline__ float row_extreme(const uint32_t (&s)[BN], bool neg) {
    float a[43];
    if (!neg) {
#pragma unroll
        for (int i = 0; i < 42; ++i)
            a[i] = max3f(__uint_as_float(s[3 * i]), __uint_as_float(s[3 * i + 1]),
                         __uint_as_float(s[3 * i + 2]));
        a[42] = fmaxf(__uint_as_float(s[126]), __uint_as_float(s[127]));
#pragma unroll
        for (int i = 0; i < 14; ++i) a[i] = max3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        a[14] = a[42];
#pragma unroll
        for (int i = 0; i < 5; ++i) a[i] = max3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        return max3f(fmaxf(a[0], a[1]), a[2], fmaxf(a[3], a[4]));
    } else {
#pragma unroll
        for (int i = 0; i < 42; ++i)
            a[i] = min3f(__uint_as_float(s[3 * i]), __uint_as_float(s[3 * i + 1]),
                         __uint_as_float(s[3 * i + 2]));
        a[42] = fminf(__uint_as_float(s[126]), __uint_as_float(s[127]));
#pragma unroll
        for (int i = 0; i < 14; ++i) a[i] = min3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        a[14] = a[42];
#pragma unroll
        for (int i = 0; i < 5; ++i) a[i] = min3f(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
        return min3f(fminf(a[0], a[1]), a[2], fminf(a[3], a[4]));
    }
}

// 2^x for a pair of x values on the FMA pipe: x = j + f with j = round(x)
// (adding 1.5 * 2^23 leaves j in the low mantissa bits), 2^f from the
// polynomial, and j added straight into the exponent field.  x is clamped to
// >= -125 so that the result stays a normal number (2^-125 is 0 for every
// practical purpose next to the row's leading term 2^0).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
    const float x0 = fmaxf(f2_lo(x), -125.f), x1 = fmaxf(f2_hi(x), -125.f);
    const uint64_t xc = f2_pack(x0, x1);
    const uint64_t big = f2_pack(12582912.f, 12582912.f);
    const uint64_t y = f2_add(xc, big);
    const uint64_t jf = f2_add(y, f2_pack(-12582912.f, -12582912.f));
    const uint64_t f = f2_add(xc, f2_pack(-f2_lo(jf), -f2_hi(jf)));
    uint64_t q = f2_fma(f2_pack(kExp2P3, kExp2P3), f, f2_pack(kExp2P2, kExp2P2));
    q = f2_fma(q, f, f2_pack(kExp2P1, kExp2P1));
    q = f2_fma(q, f, f2_pack(kExp2P0, kExp2P0));
    const uint32_t r0 = static_cast<uint32_t>(q) + (static_cast<uint32_t>(y) << 23);
    const uint32_t r1 = static_cast<uint32_t>(q >> 32) + (static_cast<uint32_t>(y >> 32) << 23);
    return (static_cast<uint64_t>(r1) << 32) | r0;
}

// p = 2^(scale*log2e*s - m) for the 128 scores of a row, packed to bf16 pairs
// in pk; returns the row sum of p.  With MASKED, keys from `lim` on give
// exactly 0.
template <bool MASKED>
__device__ __forceinline__ float exp_pairs(const uint32_t (&s)[BN], uint32_t (&pk)[BN / 2],
                                           uint64_t sl2, float m, int lim) {
    const float mb = (m == -INFINITY) ? 0.f : m;
    const uint64_t nm2 = f2_pack(-mb, -mb);
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < BN; c += 2) {
        const uint64_t x =
            f2_fma(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2, nm2);
        float p0, p1;
        if ((c / 2) % 8 < kPolyPairs) {
            const uint64_t e = exp2_poly2(x);
            p0 = f2_lo(e);
            p1 = f2_hi(e);
        } else {
            p0 = ex2_approx(f2_lo(x));
            p1 = ex2_approx(f2_hi(x));
        }
        if constexpr (MASKED) {
            p0 = (c < lim) ? p0 : 0.f;
            p1 = (c + 1 < lim) ? p1 : 0.f;
        }
        acc[(c / 2) & 3] = f2_add(acc[(c / 2) & 3], f2_pack(p0, p1));
        pk[c / 2] = pack_bf16x2(p0, p1);
    }
    const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    return f2_lo(a2) + f2_hi(a2);
}

// MODE: kFixed ([B,H,N,d] tensors), kVarlen (packed [total,H,d] sequences),
// kPaged (packed queries; keys and values read through the page table from a
// pool of 256-token pages, the queries being the last positions of each
// cached sequence).
// PAIR (fixed-length, d = 128, no RoPE): CTAs run in clusters of two and a
// pair shares one 512-row query block: CTA c of the pair holds 128-row tiles
// 2t + c (t = 0, 1), and tile pair t (rows 256t .. 256t + 255 of the block) is
// one M = 256 product on both SMs.  Each CTA loads half of every K tile (64
// keys) and half of every V tile (64 dimensions), so each K/V byte crosses
// from L2 once per 512 query rows instead of once per 256, and the B operand
// is read from shared memory once for both SMs.  The even CTA issues every
// MMA; both CTAs run the softmax and epilogue of their own tiles.
template <int D, int MODE, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const FwdParams p) {
    constexpr bool VARLEN = MODE != kFixed;  // packed query rows
    constexpr bool PAGED = MODE == kPaged;
    static_assert(!PAIR || (D == 128 && MODE == kFixed), "pair mode: fixed length, d=128");
    constexpr int R = ring_slots<PAIR>();          // K/V ring slots
    constexpr int kRows = PAIR ? 4 * BM : 2 * BM;  // query rows per work unit
    // ---- the work unit: (sequence/head, query block of kRows rows) ---------
    // CTAs (CTA pairs) walk the units in groups of kHeadGroup (sequence, head)
    // pairs; in a group they are numbered by rank first, rank r being the r-th
    // block counted from the end of its sequence.  Under a causal mask each
    // group's heaviest blocks start before its lighter ones, and the CTAs in
    // flight at any time read the K/V of a few heads only, which stay in L2
    // (all heads at once would spill it and re-read K/V from DRAM).  With
    // grouped K/V heads (H_kv < H) query head h reads K/V head h / (H / H_kv).
    const int wu = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const uint32_t crank = PAIR ? cluster_ctarank() : 0u;  // 0: issues the pair's MMAs
    const int units = p.B * p.H;
    const int nblk_all = (p.N + kRows - 1) / kRows;
    const int gidx = wu / (kHeadGroup * nblk_all);
    const int ug = min(kHeadGroup, units - gidx * kHeadGroup);
    const int within = wu - gidx * kHeadGroup * nblk_all;
    const int rank = within / ug;
    const int unit = gidx * kHeadGroup + (within - rank * ug);
    // len: query rows; klen: keys; a query row i may see keys up to
    // kshift + i under the causal mask (kshift = klen - len for paged
    // prefill, whose queries end the sequence; 0 otherwise)
    int len, klen, kshift = 0, seq_start = 0, bh = 0, h = 0, bkv = 0, b = 0;
    if constexpr (VARLEN) {
        const int bi = unit / p.H;  // the bi-th sequence to run, heaviest first
        b = p.seq_order ? p.seq_order[bi] : bi;
        h = unit - bi * p.H;
        const int s0 = p.cu_seqlens[b], s1 = p.cu_seqlens[b + 1];
        // keep every access inside the [total, H, d] tensors whatever the offsets say
        const int c0 = min(max(s0, 0), p.total), c1 = min(max(s1, c0), p.total);
        const int c1m = min(c1, c0 + p.N);
        if ((c0 != s0 || c1m != s1) && rank == 0 && h == 0 && threadIdx.x == 0)
            record_error(p.err, FA_DEVERR_BAD_INPUT);
        seq_start = c0;
        len = c1m - c0;
        klen = len;
        bkv = h / (p.H / p.H_kv);  // packed K/V: the head coordinate of the token rows
        if constexpr (PAGED) {
            const int ctx = p.ctx_lens[b];
            if (ctx < len) {  // more queries than cached tokens: not computed
                if (rank == 0 && threadIdx.x == 0) record_error(p.err, FA_DEVERR_BAD_INPUT);
                return;
            }
            klen = ctx;
            kshift = ctx - len;
        }
    } else {
        bh = unit;
        b = bh / p.H;
        bkv = b * p.H_kv + (bh - b * p.H) / (p.H / p.H_kv);
        len = p.N;
        klen = len;
    }
    const int nblk = (len + kRows - 1) / kRows;
    const int blk = p.causal ? (nblk - 1 - rank) : rank;
    if (blk < 0 || blk >= nblk) return;  // (both CTAs of a pair return together)
    const int row0 = blk * kRows;
    // first query row of this CTA's tile t
    auto tile_row = [&](int t) { return PAIR ? row0 + (2 * t + static_cast<int>(crank)) * BM
                                             : row0 + t * BM; };
    const int nkv_all = (klen + BN - 1) / BN;
    // n_t[t]: K/V tiles tile t takes part in; a pair's two tiles share one
    // count, that of its later tile (the earlier tile's last step is then
    // fully masked under a causal mask and contributes P = 0)
    int n_t[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int rf = PAIR ? row0 + 2 * t * BM : row0 + t * BM;   // first row that must be computed
        const int rl = PAIR ? rf + BM : rf;                         // first row of the last tile
        n_t[t] = (rf < len) ? (p.causal ? min((kshift + rl + BM - 1) / BN + 1, nkv_all) : nkv_all)
                            : 0;
    }
    const int n = max(n_t[0], n_t[1]);
    // paged: the last K/V tile runs past the sequence end into the rest of
    // its page; those V rows are zeroed before P V (P is 0 there, but 0 * NaN
    // would not be)
    const bool zero_v_tail = PAGED && n == nkv_all && (klen % BN) != 0;

    extern __shared__ uint8_t smem_raw[];
    FwdSmem<D, PAIR>& sm = *reinterpret_cast<FwdSmem<D, PAIR>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const uint32_t warp = warp_id_uniform();
    const uint32_t lane = lane_id();
    const uint32_t wg = warp / 4;
    unsigned int* err = p.err;
    volatile int* abort = &sm.abort;
    const uint64_t wlim = p.wait_ns ? p.wait_ns : FA_WAIT_TIMEOUT_NS;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sm.q_full[t], 1);
            mbar_init(&sm.s_full[t], 1);
            mbar_init(&sm.p_full[t], PAIR ? 8 : BM);  // pair: one arrival per softmax warp
            mbar_init(&sm.pv_done[t], 1);
            mbar_init(&sm.stats_full[t], BM);
        }
        mbar_init(&sm.vfix, 1);
        for (int s = 0; s < R; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbar_init();
    }
    if (warp == 12) {
        if constexpr (PAIR) {
            tmem_alloc_pair(&sm.tmem_base, kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&sm.tmem_base, kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    // a pair: the other CTA's barriers must be initialised before any copy,
    // commit or arrival reaches them
    if constexpr (PAIR) cluster_sync_all();
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (wg == 3) {
        regs_dec<kRegsIssue>();
        if (warp == 13) {
            // ================= TMA producer =================
            // paged: sequence b's pages start at entry sum_{b'<b} ceil(ctx_b'/256)
            int page_base = 0;
            if constexpr (PAGED) {
                for (int i = lane; i < b; i += 32) page_base += (max(p.ctx_lens[i], 0) + 255) / 256;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) page_base += __shfl_xor_sync(0xffffffffu, page_base, o);
            }
            int issued = 0;  // ring uses issued so far
            if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            // head: the fixed-length maps' outer coordinate (flat sequence/head),
            // or the packed maps' head coordinate
            auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row,
                                 int head) {
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) {
                    if constexpr (VARLEN)
                        tma_load_3d(dst + cb * kBoxBytes, map, bar, cb * 64, head, seq_start + row);
                    else
                        tma_load_3d(dst + cb * kBoxBytes, map, bar, cb * 64, row, head);
                }
            };
            // paged K/V: key tile j is the 128-slot half (j % 2) of page
            // page_table[page_base + j / 2]; the pool map is (d, slot, page*H_kv + head)
            auto load_kv = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int j) {
                const int page = p.page_table[page_base + (j >> 1)];
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load_3d(dst + cb * kBoxBytes, map, bar, cb * 64, (j & 1) * BN,
                                page * p.H_kv + bkv);
            };
            if constexpr (PAIR) {
                // Both CTAs copy into their own shared memory and complete the
                // bytes on the even CTA's barriers, whose single arrival (with
                // the byte count of both halves) the even CTA makes.
                for (int t = 0; t < 2; ++t) {
                    if (n_t[t] == 0) continue;
                    if (crank == 0) mbar_arrive_expect_tx(&sm.q_full[t], 2 * BM * D * 2);
                    const uint32_t bar = mapa_rank(smem_u32(&sm.q_full[t]), 0);
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load_3d_pair(sm.q[t] + cb * kBoxBytes, &tq, bar, cb * 64, tile_row(t),
                                         bh);
                }
                for (int u = 0; u < 2 * n; ++u) {
                    if (u + 1 == p.withhold_copy) break;  // failure-detection check
                    const int slot = u % R;
                    const uint32_t ph = (u / R) & 1;
                    if (!mbar_wait(&sm.kv_empty[slot], ph ^ 1, err, FA_DEVERR_TIMEOUT, abort, wlim)) break;
                    if (crank == 0) mbar_arrive_expect_tx(&sm.kv_full[slot], BN * D * 2);
                    const uint32_t bar = mapa_rank(smem_u32(&sm.kv_full[slot]), 0);
                    const int j = u >> 1;
                    if ((u & 1) == 0) {
                        // K: keys [j*BN + crank*BN/2, +BN/2), every dimension
                        // (D/64 boxes of BN/2 rows x 64 columns)
#pragma unroll
                        for (int cb = 0; cb < D / 64; ++cb)
                            tma_load_3d_pair(sm.kv[slot] + cb * (kBoxBytes / 2), &tk, bar, cb * 64,
                                             j * BN + static_cast<int>(crank) * (BN / 2), bkv);
                    } else {
                        // V: every key of the tile, dimensions [crank*64, +64)
                        tma_load_3d_pair(sm.kv[slot], &tv, bar, static_cast<int>(crank) * 64,
                                         j * BN, bkv);
                    }
                    issued = u + 1;
                }
            } else {
            for (int t = 0; t < 2; ++t) {
                if (n_t[t] > 0) {
                    mbar_arrive_expect_tx(&sm.q_full[t], BM * D * 2);
                    load_tile(sm.q[t], &tq, &sm.q_full[t], tile_row(t), VARLEN ? h : bh);
                }
            }
            for (int u = 0; u < 2 * n; ++u) {
                // failure-detection check: this copy (and every later one) is
                // withheld, so its consumer's bounded wait runs out
                if (u + 1 == p.withhold_copy) break;
                const int slot = u % R;
                const uint32_t ph = (u / R) & 1;
                if (!mbar_wait(&sm.kv_empty[slot], ph ^ 1, err, FA_DEVERR_TIMEOUT, abort, wlim)) break;
                mbar_arrive_expect_tx(&sm.kv_full[slot], BN * D * 2);
                if constexpr (PAGED)
                    load_kv(sm.kv[slot], (u & 1) ? &tv : &tk, &sm.kv_full[slot], u >> 1);
                else
                    load_tile(sm.kv[slot], (u & 1) ? &tv : &tk, &sm.kv_full[slot], (u >> 1) * BN,
                              bkv);
                issued = u + 1;
            }
            }  // PAIR
            }  // lane 0
            issued = __shfl_sync(0xffffffffu, issued, 0);
            if (zero_v_tail && issued == 2 * n) {
                // the whole warp: once V_{n-1} has landed, clear its rows past
                // the sequence end (whole 128-byte rows, so the swizzle does not
                // matter), make the writes visible to the tensor core, release
                const int vs = ring_slot(n - 1, 1);
                if (warp_wait(&sm.kv_full[vs], ring_phase(n - 1, 1), err, abort, wlim)) {
                    const int zr = klen - (n - 1) * BN;  // first row to clear
                    uint4* base = reinterpret_cast<uint4*>(sm.kv[vs]);
                    const int per_box = (BN - zr) * 8;   // 16-byte words per box
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb)
                        for (int i = lane; i < per_box; i += 32)
                            base[cb * (kBoxBytes / 16) + zr * 8 + i] = make_uint4(0, 0, 0, 0);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.vfix);
                }
            }
            if (lane == 0) {
            // every copy this CTA started must land before it exits
            if (crank == 0) {
                for (int t = 0; t < 2; ++t)
                    if (n_t[t] > 0) mbar_wait(&sm.q_full[t], 0, err, FA_DEVERR_TIMEOUT, nullptr, wlim);
                for (int u = max(0, issued - R); u < issued; ++u)
                    mbar_wait(&sm.kv_full[u % R], (u / R) & 1, err, FA_DEVERR_TIMEOUT, nullptr, wlim);
            } else {
                // the odd CTA of a pair cannot wait on the even CTA's barriers:
                // a slot released by the MMAs has landed (and so has Q, read
                // by earlier products)
                for (int u = max(0, issued - R); u < issued; ++u)
                    mbar_wait(&sm.kv_empty[u % R], (u / R) & 1, err, FA_DEVERR_TIMEOUT, abort, wlim);
            }
            }  // lane 0
        } else if (warp == 12 && lane == 0 && crank == 0) {
            // ================= MMA issuer =================
            // The tensor pipe runs this thread's MMAs in issue order, so
            // S_t(j+1), which overwrites the TMEM columns holding P_t(j), is
            // issued right behind P_t(j) V_j without waiting: P_t is read first.
            // A pair's products have M = 256 (this CTA's tile, then the odd
            // CTA's) and take half of B's columns from each CTA.
            constexpr uint32_t kM = PAIR ? 2 * BM : BM;
            constexpr uint32_t idesc_s = idesc_bf16_f32(kM, BN, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, D, 0, 1);
            // descriptor words: high = SBO 1024 B | version 1 | 128-byte swizzle;
            // low = LBO (16 B for K-major, the 64-column block stride for V) | addr>>4
            constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
            constexpr uint32_t kLboK = (16u >> 4) << 16;
            constexpr uint32_t kLboV = (static_cast<uint32_t>(kBoxBytes) >> 4) << 16;
            constexpr uint32_t kSlot16 = FwdSmem<D, PAIR>::kSlotBytes >> 4;  // ring slot, 16-B units
            // K in a slot: D/64 boxes of (PAIR ? 64 : 128) keys x 128 bytes
            constexpr uint32_t kKBox16 = (PAIR ? kBoxBytes / 2 : kBoxBytes) >> 4;
            const uint32_t q_lo0 = smem_u32(sm.q[0]) >> 4;
            const uint32_t q_lo1 = smem_u32(sm.q[1]) >> 4;
            const uint32_t kv_lo = smem_u32(sm.kv[0]) >> 4;
            auto issue_s = [&](int t, int j) {
                const uint32_t qa = t ? q_lo1 : q_lo0;
                const uint32_t kb = kv_lo + ring_slot<R>(j, 0) * kSlot16;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = (kk >> 2) * (kBoxBytes >> 4) + (kk & 3) * 2;
                    const uint32_t ob = (kk >> 2) * kKBox16 + (kk & 3) * 2;
                    const uint64_t da = (static_cast<uint64_t>(kDescHi) << 32) | (kLboK | (qa + oa));
                    const uint64_t db = (static_cast<uint64_t>(kDescHi) << 32) | (kLboK | (kb + ob));
                    if constexpr (PAIR)
                        mma_ss_pair(tmem + col_s(t), da, db, idesc_s, kk > 0 ? 1u : 0u);
                    else
                        mma_ss(tmem + col_s(t), da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int t, int j) {
                const uint32_t vb = kv_lo + ring_slot<R>(j, 1) * kSlot16;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {  // 16 keys = 16 rows of 128 bytes
                    const uint64_t db =
                        (static_cast<uint64_t>(kDescHi) << 32) | (kLboV | (vb + kk * 128));
                    if constexpr (PAIR)
                        mma_ts_pair(tmem + col_o(t), tmem + col_s(t) + kk * 8, db, idesc_pv,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    else
                        mma_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, db, idesc_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            // completion of everything issued so far, signalled to this CTA's
            // barrier and, for a pair, to the same barrier of the odd CTA
            auto commit = [&](uint64_t* bar) {
                if constexpr (PAIR) {
                    tc_commit_pair(smem_u32(bar));
                    tc_commit_pair(mapa_rank(smem_u32(bar), 1));
                } else {
                    tc_commit(bar);
                }
            };
            bool ok = true;
            auto wait_k = [&](int j) {
                return mbar_wait(&sm.kv_full[ring_slot<R>(j, 0)], ring_phase<R>(j, 0), err,
                                 FA_DEVERR_TIMEOUT, abort, wlim);
            };
            for (int t = 0; t < 2 && ok; ++t)
                if (n_t[t] > 0)
                    ok = mbar_wait(&sm.q_full[t], 0, err, FA_DEVERR_TIMEOUT, abort, wlim);
            ok = ok && wait_k(0);
            if (ok) {
                tc_fence_after();
                for (int t = 0; t < 2; ++t) {
                    if (n_t[t] > 0) {
                        issue_s(t, 0);
                        commit(&sm.s_full[t]);
                    }
                }
                commit(&sm.kv_empty[ring_slot<R>(0, 0)]);
            }
            for (int j = 0; ok && j < n; ++j) {
                if (zero_v_tail && j == n - 1) {
                    if (!mbar_wait(&sm.vfix, 0, err, FA_DEVERR_TIMEOUT, abort, wlim)) break;
                } else if (!mbar_wait(&sm.kv_full[ring_slot<R>(j, 1)], ring_phase<R>(j, 1), err,
                                      FA_DEVERR_TIMEOUT, abort, wlim)) {
                    break;
                }
                const bool next_k = j + 1 < n;
                if (next_k && !wait_k(j + 1)) break;
                for (int t = 0; t < 2; ++t) {
                    if (j >= n_t[t]) continue;
                    // a pair's P comes from both CTAs' softmax warps
                    if (!mbar_wait<PAIR>(&sm.p_full[t], j & 1, err, FA_DEVERR_TIMEOUT, abort, wlim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(t, j);
                    if (j + 1 == n_t[t]) commit(&sm.pv_done[t]);  // O_t final
                    if (j + 1 < n_t[t]) {
                        issue_s(t, j + 1);
                        commit(&sm.s_full[t]);
                    }
                }
                if (!ok) break;
                commit(&sm.kv_empty[ring_slot<R>(j, 1)]);
                if (next_k) commit(&sm.kv_empty[ring_slot<R>(j + 1, 0)]);
            }
            // every MMA this thread issued must be complete before TMEM is freed
            if constexpr (PAIR) tc_commit_pair(smem_u32(&sm.drain));
            else tc_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, err, FA_DEVERR_TIMEOUT, nullptr, wlim);
        }
        __syncwarp();
    } else if (wg < 2) {
        // ================= softmax of tile t (warpgroups 0 and 1) =================
        regs_inc<kRegsSoftmax>();
        const int t = wg;
        const int r = threadIdx.x - t * BM;          // row within the tile == TMEM lane
        const uint32_t lane_off = ((warp & 3) * 32u) << 16;
        const uint32_t s_addr = tmem + lane_off + col_s(t);
        const uint32_t o_addr = tmem + lane_off + col_o(t);
        const int row_first = tile_row(t);
        const int qrow = row_first + r;
        const float sl = p.scale_log2;
        const bool neg = sl < 0.f;
        const uint64_t sl2 = f2_pack(sl, sl);
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_t[t]; ++j) {
            if (!warp_wait(&sm.s_full[t], j & 1, err, abort, wlim)) { ok = false; break; }
            tc_fence_after();
            // masked keys: past the sequence end, or after this row (causal)
            const int kbase = j * BN;
            const bool need_mask =
                (kbase + BN > klen) || (p.causal && kbase + BN - 1 > kshift + row_first);
            int lim = BN;
            if (need_mask) {
                lim = min(BN, klen - kbase);
                if (p.causal) lim = min(lim, kshift + qrow - kbase + 1);
            }
            uint32_t s[BN];
            uint32_t pk[BN / 2];
            float alpha = 1.f, rs = 0.f;
            // Pass 1 uses the running max of earlier steps; if that leaves a
            // row sum above kLazySum anywhere in the warp (or on the first
            // step), pass 2 reloads the scores and uses the true row max.
            for (int pass = (j == 0) ? 1 : 0; pass < 2; ++pass) {
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
                tmem_wait_ld();
                if (need_mask) {
                    const uint32_t fill = __float_as_uint(neg ? INFINITY : -INFINITY);
#pragma unroll
                    for (int c = 0; c < BN; ++c) s[c] = (c < lim) ? s[c] : fill;
                }
                if (pass == 1) {
                    const float mt = row_extreme(s, neg) * sl;  // max over keys of scale*log2e*s
                    if (j == 0) {
                        m_used = mt;
                    } else if (mt > m_used) {
                        alpha = ex2_approx(m_used - mt);
                        m_used = mt;
                    }
                }
                rs = need_mask ? exp_pairs<true>(s, pk, sl2, m_used, lim)
                               : exp_pairs<false>(s, pk, sl2, m_used, BN);
                if (pass == 1 || !__any_sync(0xffffffffu, !(rs <= kLazySum))) break;
            }
            l = l * alpha + rs;
            tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            // O_t holds P_t V_0..j-1 and is idle: S_t(j) was issued behind
            // P_t V_{j-1} in the MMA stream, so that product has completed.
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    const uint32_t addr = o_addr + c * 32;
                    tmem_ld32(addr, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint64_t v = f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
                        o[e] = static_cast<uint32_t>(v);
                        o[e + 1] = static_cast<uint32_t>(v >> 32);
                    }
                    tmem_st32(addr, o);
                }
            }

            tmem_wait_st();
            tc_fence_before();
            if constexpr (PAIR) {
                // one arrival per warp on the even CTA's barrier
                __syncwarp();
                if (lane == 0) {
                    if (crank == 0) mbar_arrive(&sm.p_full[t]);
                    else mbar_arrive_cluster(mapa_rank(smem_u32(&sm.p_full[t]), 0));
                }
            } else {
                mbar_arrive(&sm.p_full[t]);
            }
        }
        if (ok && n_t[t] > 0) {
            sm.row_m[t][r] = m_used;
            sm.row_l[t][r] = l;
            mbar_arrive(&sm.stats_full[t]);
        }
    } else {
        // ================= epilogue (warpgroup 2) =================
        regs_dec<kRegsEpilogue>();
        const int r = threadIdx.x - 2 * BM;
        const uint32_t lane_off = ((warp & 3) * 32u) << 16;
        bool ok = true;
        // epilogue: O / l -> bf16, log-sum-exp
        for (int t = 0; ok && t < 2; ++t) {
            if (n_t[t] == 0) continue;
            if (!warp_wait(&sm.stats_full[t], 0, err, abort, wlim) ||
                !warp_wait(&sm.pv_done[t], 0, err, abort, wlim))
                break;
            tc_fence_after();
            const int qrow = tile_row(t) + r;
            const bool store = qrow < len;
            const float m = sm.row_m[t][r], l = sm.row_l[t][r];
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
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + col_o(t) + c * 32, o);
                tmem_wait_ld();
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[e * 8 + 0]) * inv_l,
                                          __uint_as_float(o[e * 8 + 1]) * inv_l);
                        w.y = pack_bf16x2(__uint_as_float(o[e * 8 + 2]) * inv_l,
                                          __uint_as_float(o[e * 8 + 3]) * inv_l);
                        w.z = pack_bf16x2(__uint_as_float(o[e * 8 + 4]) * inv_l,
                                          __uint_as_float(o[e * 8 + 5]) * inv_l);
                        w.w = pack_bf16x2(__uint_as_float(o[e * 8 + 6]) * inv_l,
                                          __uint_as_float(o[e * 8 + 7]) * inv_l);
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
    // a pair: neither CTA may free its TMEM or leave (its shared memory still
    // read by the pair's products, its barriers still arrived on) before both
    // are done
    if constexpr (PAIR) cluster_sync_all();
    else __syncthreads();
    tc_fence_after();
    if (warp == 12) {
        if constexpr (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
        else tmem_dealloc(tmem, kTmemCols);
    }
}

// Rotary position embedding of whole rows in device memory, applied once per
// position before the attention (the page "“Flash”不是那个被时代淘汰的插件"
// (0539edu.com): the kernel fuses RoPE, section 2, from a precomputed sin/cos
// lookup table, section 3): rows x0 [rows0, N, D] -> y0 and x1 [rows1, N, D]
// -> y1 in one launch, row n at position n.  Pairs (i, i + D/2) are turned by
// the angle whose cosine and sine are cos_t[pos*(D/2) + i], sin_t[...]:
// x_i cos - x_{i+D/2} sin and x_{i+D/2} cos + x_i sin, every product and sum
// rounded to fp32 (no fused multiply-add: a fixed, reproducible order), then
// rounded to bf16 for the tensor cores.  One thread per (two rows, position,
// 8 pairs): the rows share the table entries (the pass reads half the table
// bytes) and both rows' loads are in flight together (about 10 us faster per
// launch on the long-prefill workload than one row per thread).
template <int D>
__global__ void __launch_bounds__(256)
    fa_rope_rows_kernel(const __nv_bfloat16* __restrict__ x0, __nv_bfloat16* __restrict__ y0,
                        int64_t rows0, const __nv_bfloat16* __restrict__ x1,
                        __nv_bfloat16* __restrict__ y1, int64_t rows1,
                        const float* __restrict__ cos_t, const float* __restrict__ sin_t, int N) {
    constexpr int HALF = D / 2, G = HALF / 8;  // 8-pair groups per row
    // an item: rows 2r and 2r + 1 (the latter if it exists) of one tensor at
    // one position and one group of 8 pairs; the two rows share the table
    // entries, and both rows' loads are issued before either is computed
    const int64_t pairs0 = (rows0 + 1) / 2, pairs1 = (rows1 + 1) / 2;
    const int64_t n0 = pairs0 * N * G;
    const int64_t total = n0 + pairs1 * N * G;
    for (int64_t wi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; wi < total;
         wi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool second = wi >= n0;
        const int64_t w = second ? wi - n0 : wi;
        const int64_t rows = second ? rows1 : rows0;
        const int g = static_cast<int>(w % G);
        const int64_t rn = w / G;  // flat (row pair, position)
        const int pos = static_cast<int>(rn % N);
        const int64_t r0 = 2 * (rn / N);
        const bool has1 = r0 + 1 < rows;
        const __nv_bfloat16* xs = second ? x1 : x0;
        __nv_bfloat16* ys = second ? y1 : y0;
        const int64_t o0 = (r0 * N + pos) * D + 8 * g;
        const int64_t o1 = has1 ? o0 + static_cast<int64_t>(N) * D : o0;
        uint4 ua[2], ub[2];
        ua[0] = *reinterpret_cast<const uint4*>(xs + o0);
        ub[0] = *reinterpret_cast<const uint4*>(xs + o0 + HALF);
        ua[1] = *reinterpret_cast<const uint4*>(xs + o1);
        ub[1] = *reinterpret_cast<const uint4*>(xs + o1 + HALF);
        const float* ct = cos_t + static_cast<int64_t>(pos) * HALF + 8 * g;
        const float* st = sin_t + static_cast<int64_t>(pos) * HALF + 8 * g;
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(ct));
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(ct + 4));
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(st));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(st + 4));
        const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int it = 0; it < 2; ++it) {
            if (it == 1 && !has1) break;
            const uint32_t wa[4] = {ua[it].x, ua[it].y, ua[it].z, ua[it].w};
            const uint32_t wb[4] = {ub[it].x, ub[it].y, ub[it].z, ub[it].w};
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a[2] = {__uint_as_float(wa[e] << 16), __uint_as_float(wa[e] & 0xffff0000u)};
                const float bb[2] = {__uint_as_float(wb[e] << 16), __uint_as_float(wb[e] & 0xffff0000u)};
                float ra[2], rb[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float cc = cs[2 * e + k], ss = sn[2 * e + k];
                    ra[k] = __fsub_rn(__fmul_rn(a[k], cc), __fmul_rn(bb[k], ss));
                    rb[k] = __fadd_rn(__fmul_rn(bb[k], cc), __fmul_rn(a[k], ss));
                }
                oa[e] = pack_bf16x2(ra[0], ra[1]);
                ob[e] = pack_bf16x2(rb[0], rb[1]);
            }
            __nv_bfloat16* dst = ys + (it ? o1 : o0);
            *reinterpret_cast<uint4*>(dst) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
            *reinterpret_cast<uint4*>(dst + HALF) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
    }
}

template <int D, int MODE, bool PAIR = false>
int launch_impl(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, cudaStream_t stream) {
    // Every CTA allocates all 512 TMEM columns, so one CTA per SM: ask for
    // enough shared memory that a second CTA cannot be co-resident.
    constexpr size_t kSmemUse = sizeof(FwdSmem<D, PAIR>) + 1024;
    const size_t smem = kSmemUse > 120 * 1024 ? kSmemUse : 120 * 1024;
    auto kern = fa_fwd_kernel<D, MODE, PAIR>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FA_ERR_CUDA;
    // one CTA (pair) per (sequence/head, query block); see the kernel for the order
    constexpr int kRows = PAIR ? 4 * BM : 2 * BM;
    const long long blocks = (p.N + kRows - 1) / kRows;
    const long long ctas = blocks * p.B * p.H * (PAIR ? 2 : 1);
    if (ctas > 0x7fffffffLL) return FA_ERR_SHAPE;
    if constexpr (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ctas));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p) != cudaSuccess) {
            cudaGetLastError();
            return FA_ERR_CUDA;
        }
        return FA_OK;
    } else {
        kern<<<dim3(static_cast<unsigned>(ctas)), kThreads, smem, stream>>>(tq, tk, tv, p);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
}

// The packed sequences by decreasing work, one CTA: work = attended (query,
// key) pairs (causal: row i sees kshift + i + 1 keys); rank = how many
// sequences come before (more work, or as much and a lower index).  The
// forward pass then starts its heaviest sequences first, and the lighter ones
// fill the last wave (longest-processing-time-first list scheduling).
__global__ void __launch_bounds__(1024)
    fa_seq_order_kernel(const int32_t* __restrict__ cu_seqlens,
                        const int32_t* __restrict__ ctx_lens, int B, int causal,
                        int32_t* __restrict__ order) {
    __shared__ long long work[kSeqOrderMax];
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const long long len = max(0, cu_seqlens[b + 1] - cu_seqlens[b]);
        const long long klen = ctx_lens ? max(0, ctx_lens[b]) : len;
        long long w;
        if (!causal) {
            w = len * klen;
        } else {
            const long long kshift = klen - len;  // < 0 only for bad input (not computed)
            w = kshift < 0 ? 0 : len * kshift + len * (len + 1) / 2;
        }
        work[b] = w;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const long long w = work[b];
        int r = 0;
        for (int j = 0; j < B; ++j) {
            const long long x = work[j];
            r += (x > w || (x == w && j < b)) ? 1 : 0;
        }
        order[r] = b;
    }
}

}  // namespace

int launch_rope_rows(const void* x0, void* y0, int64_t rows0, const void* x1, void* y1,
                     int64_t rows1, const float* cos_t, const float* sin_t, int N, int d,
                     int num_sms, cudaStream_t stream) {
    using T = __nv_bfloat16;
    if (d == 128)
        fa_rope_rows_kernel<128><<<num_sms * 8, 256, 0, stream>>>(
            static_cast<const T*>(x0), static_cast<T*>(y0), rows0, static_cast<const T*>(x1),
            static_cast<T*>(y1), rows1, cos_t, sin_t, N);
    else if (d == 64)
        fa_rope_rows_kernel<64><<<num_sms * 8, 256, 0, stream>>>(
            static_cast<const T*>(x0), static_cast<T*>(y0), rows0, static_cast<const T*>(x1),
            static_cast<T*>(y1), rows1, cos_t, sin_t, N);
    else
        return FA_ERR_UNSUPPORTED;
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int launch_fwd(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
               const CUtensorMap& tv, int d, int mode, cudaStream_t stream) {
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    switch (mode) {
        case kFixedPair:
            if (d != 128) return FA_ERR_UNSUPPORTED;
            return launch_impl<128, kFixed, true>(p, tq, tk, tv, stream);
        case kFixed:
            return d == 128 ? launch_impl<128, kFixed>(p, tq, tk, tv, stream)
                            : launch_impl<64, kFixed>(p, tq, tk, tv, stream);
        case kVarlen:
            return d == 128 ? launch_impl<128, kVarlen>(p, tq, tk, tv, stream)
                            : launch_impl<64, kVarlen>(p, tq, tk, tv, stream);
        case kPaged:
            return d == 128 ? launch_impl<128, kPaged>(p, tq, tk, tv, stream)
                            : launch_impl<64, kPaged>(p, tq, tk, tv, stream);
        default: return FA_ERR_UNSUPPORTED;
    }
}

int launch_seq_order(const int32_t* cu_seqlens, const int32_t* ctx_lens, int B, int causal,
                     int32_t* order, cudaStream_t stream) {
    if (B < 1 || B > kSeqOrderMax) return FA_ERR_SHAPE;
    fa_seq_order_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, ctx_lens, B, causal, order);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
