// decode_sm100.cu -- single-token decode over a paged KV cache, and the gather
// of a paged cache back into contiguous rows.
//
// The cache is the fixed page pool of the page "“Flash”不是那个被时代淘汰的插件"
// (0539edu.com), section 2: pages of 256 tokens, each a contiguous K (or V)
// slice, handed to sequences from the pool.  The same section notes that
// decode is bound by memory traffic rather than arithmetic, so this path is
// written for HBM bandwidth: every K/V byte is read exactly once with 128-bit
// coalesced loads, and the tensor cores are not used (one query row per
// head gives a matrix-vector product).
//
// Decode runs as three launches on the caller's stream:
//   plan   -- one CTA: prefix sums over the sequences of pages, tokens and
//             work units (a unit is one head of one split of one sequence);
//   split  -- a persistent grid, one CTA per SM, over the units; a unit
//             attends its query to the tokens of a few consecutive pages with
//             the online softmax (running max and normaliser, page "Flash
//             Attention 是什么", section 关键术语解析, item 4) and writes a
//             normalised partial output and its log-sum-exp.  A producer warp
//             streams each (page, head) slice -- contiguous in the pool --
//             into a 6-stage shared-memory ring with bulk copies, so each SM
//             keeps ~200 KB of reads in flight; eight consumer warps compute
//             from shared memory;
//   merge  -- per (sequence, head), the log-sum-exp merge of the partials:
//             lse = M + log sum_s 2^(lse_s - M), o = sum_s 2^(lse_s - lse) o_s.
// All logs and exponents are base 2 inside the path (scale * log2 e folded
// into the query).
#include <cuda_bf16.h>

#include <type_traits>

#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kPlanThreads = 1024;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WorkspaceLayout {
    size_t plan_bytes, lse_off, o_off, total;
};

__host__ __device__ inline WorkspaceLayout layout_of(int B, int H, int d, int max_splits) {
    WorkspaceLayout L;
    const size_t units = static_cast<size_t>(B) * H * max_splits;
    L.plan_bytes = align256(sizeof(int32_t) * 3 * (static_cast<size_t>(B) + 1));
    L.lse_off = L.plan_bytes;
    L.o_off = L.lse_off + align256(sizeof(float) * units);
    L.total = L.o_off + sizeof(float) * units * d;
    return L;
}

// Splits of a sequence with np pages: at least min_pages pages each, at most
// max_splits of them, none empty.
__device__ __forceinline__ void split_shape(int np, int max_splits, int min_pages, int& ns,
                                            int& cp) {
    if (np <= 0) {
        ns = 0;
        cp = 1;
        return;
    }
    int want = (np + min_pages - 1) / min_pages;
    if (want > max_splits) want = max_splits;
    cp = (np + want - 1) / want;
    ns = (np + cp - 1) / cp;
}

// Block-wide inclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_incl_scan(int v, int* sh /*[32]*/, int& total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) sh[w] = v;
    __syncthreads();
    if (w == 0) {
        int x = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        sh[lane] = x;
    }
    __syncthreads();
    if (w > 0) v += sh[w - 1];
    total = sh[31];
    __syncthreads();
    return v;
}

__global__ void __launch_bounds__(kPlanThreads)
    fa_decode_plan_kernel(const int32_t* __restrict__ seq_lens, int B, int H, int page_size,
                          int max_splits, int min_pages, int32_t* page_off, int32_t* tok_off,
                          int32_t* unit_off, unsigned int* err) {
    __shared__ int sh[3][32];
    int carry_p = 0, carry_t = 0, carry_u = 0;
    if (threadIdx.x == 0) {
        page_off[0] = 0;
        tok_off[0] = 0;
        unit_off[0] = 0;
    }
    for (int base = 0; base < B; base += kPlanThreads) {
        const int i = base + threadIdx.x;
        int len = 0;
        if (i < B) {
            len = seq_lens[i];
            if (len < 0) {
                record_error(err, FA_DEVERR_BAD_INPUT);
                len = 0;
            }
        }
        const int np = (len + page_size - 1) / page_size;
        int ns, cp;
        split_shape(np, max_splits, min_pages, ns, cp);
        int tp, tt, tu;
        const int ip = block_incl_scan(np, sh[0], tp);
        const int it = block_incl_scan(len, sh[1], tt);
        const int iu = block_incl_scan(ns * H, sh[2], tu);
        if (i < B) {
            page_off[i + 1] = carry_p + ip;
            tok_off[i + 1] = carry_t + it;
            unit_off[i + 1] = carry_u + iu;
        }
        carry_p += tp;
        carry_t += tt;
        carry_u += tu;
    }
}

// A block table [B, max_pages] (sequence b's k-th page at row b, entry k)
// turned into what the decode kernels read: the used entries of every row,
// back to back (the packed table), and the lengths.  A negative length is
// reported and taken as 0; a length beyond its row (max_pages * page_size
// tokens) is reported and cut to the row, so no entry outside the table is
// read.  One CTA.
__global__ void __launch_bounds__(kPlanThreads)
    fa_decode_pack_kernel(const int32_t* __restrict__ block_table, int max_pages,
                          const int32_t* __restrict__ seq_lens, int B, int page_size,
                          int32_t* __restrict__ packed, int32_t* __restrict__ lens,
                          unsigned int* err) {
    __shared__ int sh[32];
    const int64_t cap = static_cast<int64_t>(max_pages) * page_size;
    int carry = 0;
    for (int base = 0; base < B; base += kPlanThreads) {
        const int i = base + threadIdx.x;
        int len = 0;
        if (i < B) {
            len = seq_lens[i];
            if (len < 0) {
                record_error(err, FA_DEVERR_BAD_INPUT);
                len = 0;
            } else if (len > cap) {
                record_error(err, FA_DEVERR_BAD_INPUT);
                len = static_cast<int>(cap);
            }
        }
        const int np = (len + page_size - 1) / page_size;
        int tot;
        const int inc = block_incl_scan(np, sh, tot);
        if (i < B) {
            lens[i] = len;
            const int32_t* row = block_table + static_cast<int64_t>(i) * max_pages;
            int32_t* dst = packed + carry + inc - np;
            for (int k = 0; k < np; ++k) dst[k] = __ldg(row + k);
        }
        carry += tot;
    }
}

// Largest b in [0, B) with off[b] <= x (off non-decreasing, off[0] = 0).
__device__ __forceinline__ int find_owner(const int32_t* off, int B, int x) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(off + mid) <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

constexpr int kDecTok = 64;           // tokens per ring stage (a quarter of a page)
constexpr int kDecConsumerWarps = 8;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;  // + one producer warp

// Multi-head decode (one query head per K/V head): a token row is spread
// over LPT lanes (16 bytes each), G token groups per CTA.
template <int D>
struct DecSmem {
    static constexpr int LPT = D / 8;                              // lanes per token
    static constexpr int G = kDecConsumerWarps * 32 / LPT;         // token groups
    static constexpr int STAGES = 6;                               // ring depth
    alignas(128) uint8_t k[STAGES][kDecTok * D * 2];
    alignas(128) uint8_t v[STAGES][kDecTok * D * 2];
    float cm[2][G], cl[2][G];  // per-group partial state, by unit parity
    float co[2][G][D];
    uint64_t full[STAGES], empty[STAGES], cmb[2];
    int abort;
};

// Walks the units u = first, first + stride, ... in increasing order and keeps
// track of the owning sequence without a search per unit.
struct UnitCursor {
    int b = 0, next_off = 0;
    __device__ __forceinline__ void seek(const int32_t* unit_off, int B, int u) {
        while (b + 1 < B && u >= next_off) {
            ++b;
            next_off = __ldg(unit_off + b + 1);
        }
    }
};

struct UnitShape {
    int b, s, h, tok0, ntok, cp, pt_base;  // h: the unit's K/V head
};

// Units of a sequence are (split, K/V head) pairs, split-major; Hk is the
// number of K/V heads.
__device__ __forceinline__ UnitShape unit_shape(int u, UnitCursor& cur,
                                                const int32_t* __restrict__ unit_off,
                                                const int32_t* __restrict__ page_off,
                                                const int32_t* __restrict__ seq_lens, int B,
                                                int Hk, int page_size, int max_splits,
                                                int min_pages) {
    cur.seek(unit_off, B, u);
    UnitShape us;
    us.b = cur.b;
    const int r = u - __ldg(unit_off + us.b);
    us.s = r / Hk;
    us.h = r % Hk;
    int len = __ldg(seq_lens + us.b);
    if (len < 0) len = 0;
    const int np = (len + page_size - 1) / page_size;
    int ns;
    split_shape(np, max_splits, min_pages, ns, us.cp);
    us.tok0 = us.s * us.cp * page_size;
    us.ntok = min(len, us.tok0 + us.cp * page_size) - us.tok0;
    us.pt_base = __ldg(page_off + us.b) + us.s * us.cp;
    return us;
}

// One unit per (split, head); the partial output of unit u is row u.  A page
// index outside [0, num_pages) is reported and page 0 is read in its place
// (nothing outside the pool is touched; that sequence's output is garbage).
template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ k_pages,
                           const __nv_bfloat16* __restrict__ v_pages,
                           const int32_t* __restrict__ page_table,
                           const int32_t* __restrict__ seq_lens, int B, int H, int num_pages,
                           int page_size, int max_splits, int min_pages,
                           const int32_t* __restrict__ page_off,
                           const int32_t* __restrict__ unit_off, float* __restrict__ part_lse,
                           float* __restrict__ part_o, float scale_log2, unsigned int* err) {
    using Sm = DecSmem<D>;
    constexpr int LPT = Sm::LPT, G = Sm::G;
    constexpr int kDecStages = Sm::STAGES;
    constexpr int GPW = 32 / LPT;  // token groups per warp
    constexpr uint32_t kChunkBytes = kDecTok * D * 2;
    extern __shared__ uint8_t dec_smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 127) &
                                    ~static_cast<uintptr_t>(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], kDecConsumerWarps);
        }
        mbar_init(&sm.cmb[0], kDecConsumerWarps * 32);
        mbar_init(&sm.cmb[1], kDecConsumerWarps * 32);
        sm.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int total_units = __ldg(unit_off + B);
    UnitCursor cur;
    cur.next_off = (B > 1) ? __ldg(unit_off + 1) : 0x7fffffff;

    if (warp == kDecConsumerWarps) {
        // ================= producer: bulk copies of (page, head) slices =================
        int g = 0;  // ring uses so far
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
            const UnitShape us = unit_shape(u, cur, unit_off, page_off, seq_lens, B, H,
                                            page_size, max_splits, min_pages);
            const int nchunks = (us.ntok + kDecTok - 1) / kDecTok;
            constexpr int per_page = 256 / kDecTok;  // page_size is 256
            int page = 0;
            for (int c = 0; c < nchunks; ++c, ++g) {
                if (c % per_page == 0) {
                    page = __ldg(page_table + us.pt_base + c / per_page);
                    if (page < 0 || page >= num_pages) {
                        if (lane == 0) record_error(err, FA_DEVERR_BAD_INPUT);
                        page = 0;
                    }
                }
                const int slot = g % kDecStages;
                if (lane == 0) {
                    if (!mbar_wait(&sm.empty[slot], ((g / kDecStages) & 1) ^ 1, err,
                                   FA_DEVERR_TIMEOUT, abort)) {
                        ok = false;
                    } else {
                        const int64_t row = (static_cast<int64_t>(page) * H + us.h) * page_size +
                                            (c % per_page) * kDecTok;
                        mbar_arrive_expect_tx(&sm.full[slot], 2 * kChunkBytes);
                        bulk_load(sm.k[slot], k_pages + row * D, kChunkBytes, &sm.full[slot]);
                        bulk_load(sm.v[slot], v_pages + row * D, kChunkBytes, &sm.full[slot]);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        // every copy this CTA started must land before it exits
        if (lane == 0)
            for (int i = max(0, g - kDecStages); i < g; ++i)
                mbar_wait(&sm.full[i % kDecStages], (i / kDecStages) & 1, err, FA_DEVERR_TIMEOUT,
                          nullptr);
        __syncwarp();
    } else {
        // ================= consumers =================
        const int sub = lane / LPT;            // group within the warp
        const int gl = lane % LPT;             // lane within the group
        const int grp = warp * GPW + sub;      // group within the CTA
        const unsigned gmask = (LPT == 32) ? 0xffffffffu : (((1u << LPT) - 1u) << (sub * LPT));
        int g = 0, k = 0;  // ring uses, units done
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x, ++k) {
            const UnitShape us = unit_shape(u, cur, unit_off, page_off, seq_lens, B, H,
                                            page_size, max_splits, min_pages);
            float qf[8];
            {
                const uint4 qu = *reinterpret_cast<const uint4*>(
                    q + (static_cast<int64_t>(us.b) * H + us.h) * D + gl * 8);
                bf16x8_to_f32(qu, qf);
#pragma unroll
                for (int i = 0; i < 8; ++i) qf[i] *= scale_log2;
            }
            float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            const int nchunks = (us.ntok + kDecTok - 1) / kDecTok;
            for (int c = 0; c < nchunks; ++c, ++g) {
                const int slot = g % kDecStages;
                if (!mbar_wait(&sm.full[slot], (g / kDecStages) & 1, err, FA_DEVERR_TIMEOUT,
                               abort)) {
                    ok = false;
                    break;
                }
                constexpr int TPG = kDecTok / G;  // tokens per group per chunk
                float sc[TPG];
                const int base = c * kDecTok;
#pragma unroll
                for (int x = 0; x < TPG; ++x) {
                    const int t = grp + x * G;
                    const uint4 kr = *reinterpret_cast<const uint4*>(sm.k[slot] + t * D * 2 + gl * 16);
                    float kf[8];
                    bf16x8_to_f32(kr, kf);
                    float dot = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], kf[i], dot);
#pragma unroll
                    for (int o = LPT / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(gmask, dot, o);
                    sc[x] = (base + t < us.ntok) ? dot : -INFINITY;
                }
                float mb = sc[0];
#pragma unroll
                for (int x = 1; x < TPG; ++x) mb = fmaxf(mb, sc[x]);
                const float m_new = fmaxf(m, mb);
                if (m_new != -INFINITY) {
                    const float alpha = ex2_approx(m - m_new);  // m = -inf -> 0
                    l *= alpha;
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
                    for (int x = 0; x < TPG; ++x) {
                        const int t = grp + x * G;
                        if (base + t < us.ntok) {
                            const float pw = ex2_approx(sc[x] - m_new);
                            l += pw;
                            const uint4 vr =
                                *reinterpret_cast<const uint4*>(sm.v[slot] + t * D * 2 + gl * 16);
                            float vf[8];
                            bf16x8_to_f32(vr, vf);
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[i] = fmaf(pw, vf[i], acc[i]);
                        }
                    }
                    m = m_new;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[slot]);
            }
            if (!ok) break;
            // combine the G groups of this unit (buffers double-buffered by unit parity)
            const int par = k & 1;
            if (gl == 0) {
                sm.cm[par][grp] = m;
                sm.cl[par][grp] = l;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) sm.co[par][grp][gl * 8 + i] = acc[i];
            mbar_arrive(&sm.cmb[par]);
            if (!mbar_wait(&sm.cmb[par], (k >> 1) & 1, err, FA_DEVERR_TIMEOUT, abort)) {
                ok = false;
                break;
            }
            if (threadIdx.x < D) {
                float M = -INFINITY;
#pragma unroll
                for (int gi = 0; gi < G; ++gi) M = fmaxf(M, sm.cm[par][gi]);
                float L = 0.f, o = 0.f;
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    const float w = (sm.cm[par][gi] == -INFINITY) ? 0.f : ex2_approx(sm.cm[par][gi] - M);
                    L += w * sm.cl[par][gi];
                    o += w * sm.co[par][gi][threadIdx.x];
                }
                part_o[static_cast<int64_t>(u) * D + threadIdx.x] = o / L;
                if (threadIdx.x == 0) part_lse[u] = M + __log2f(L);
            }
        }
    }
}


// ---------------------------------------------------------------------------
// Grouped query heads (groups of 2 or more; see below for the sizes).  A
// unit is (split,
// K/V head); the GH query heads of its group are the rows of a 16-row MMA
// tile (rows GH..15 are zero), so each staged K/V byte serves all of them and the
// dot products run as two small matrix products per chunk on the tensor
// cores (warp-level m16n8k16: a tcgen05 tile has at least 64 rows, 8x-32x
// more than the group has).  K/V chunks of 64 tokens arrive by TMA in the
// 128-byte-swizzled layout, so the ldmatrix reads of 8 token rows at one
// column fall in 8 distinct bank groups.  Two teams of four warps take
// alternate chunks; warp wt of a team owns tokens 16wt .. 16wt+15:
//   S  = Q_g K^T   two 8-token n-tiles over D/16 k-steps (fp32)
//   online softmax per query row (rows lane / 4 and, for groups of 16,
//   lane / 4 + 8; the 4 lanes of a quad share them), base 2 with
//   scale * log2(e) applied to S
//   O += P V       P from S's accumulators as the A operand, V through
//                  ldmatrix.trans, D/8 n-tiles
// and the 8 warps' (m, l, O) are merged per unit through one shared buffer
// (a second barrier tells the writers of the next unit that every reader of
// this one is done), which leaves room for more ring stages.
// A unit holds gr <= GH query heads (GH, the template, is the capacity of
// its registers and merge buffer).  Groups larger than 16 (multi-query
// attention with many heads) are cut into equal sub-groups of gr <= 16 query
// heads.  With teams == 2 a unit holds two sub-groups of the same K/V head:
// each team of four warps takes every chunk for its own sub-group's rows, so
// a staged K/V chunk serves 2 gr query heads and is read from memory once
// for both (an even number of sub-groups is paired this way).  Otherwise
// (teams == 1) each sub-group is a unit of its own and the two teams take
// alternate chunks.  Hk counts the units per split (H / (teams gr)) and sub
// the units per K/V head: the unit's K/V head is h / sub.
// ---------------------------------------------------------------------------
constexpr int kGqTok = 64;          // tokens per chunk
constexpr int kGqWarps = 8;         // consumer warps (two teams of four)
constexpr int kGqThreads = (kGqWarps + 1) * 32;
constexpr int kGqSmemLimit = 232448;  // opt-in shared memory per block

template <int D, int GH>
struct GqSmem {
    static constexpr int kTile = kGqTok * D * 2;   // one of K, V per stage
    static constexpr int kCo = GH * kGqWarps * D * 4;
    static constexpr int kFit = (kGqSmemLimit - 2048 - 1024 - kCo) / (2 * kTile);
    // even: chunk g goes to team g % 2 and stage g % STAGES, so each stage
    // belongs to one team, which then sees every phase of its barriers in
    // order (with an odd count a team could wait on a stage two phases ahead
    // of it, and a parity wait cannot tell those phases apart)
    static constexpr int STAGES = (kFit < 6 ? kFit : 6) & ~1;
    alignas(1024) uint8_t k[STAGES][kTile];
    alignas(1024) uint8_t v[STAGES][kTile];
    // per-warp partial state of the unit being merged; cmb: every consumer
    // has written its state, cfree: every consumer has read the merged unit
    float co[GH][kGqWarps][D];
    float cm[GH][kGqWarps], cl[GH][kGqWarps];
    uint64_t full[STAGES], empty[STAGES], cmb, cfree;
    int abort;
};

// Byte offset of (token t, 16-byte column chunk c) in a staged tile: D/64
// TMA boxes of 64 rows x 128 bytes, chunk index XOR (row % 8) inside a box.
__device__ __forceinline__ uint32_t gq_swz(int t, int c) {
    return static_cast<uint32_t>((c >> 3) * (kGqTok * 128) + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

template <int D, int GH>
__global__ void __launch_bounds__(kGqThreads, 1)
    fa_decode_gqa_kernel(const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv,
                         const __nv_bfloat16* __restrict__ q,
                         const int32_t* __restrict__ page_table,
                         const int32_t* __restrict__ seq_lens, int B, int H, int Hk, int gr, int sub,
                         int teams, int num_pages, int max_splits, int min_pages,
                         const int32_t* __restrict__ page_off,
                         const int32_t* __restrict__ unit_off, float* __restrict__ part_lse,
                         float* __restrict__ part_o, float scale_log2, unsigned int* err) {
    using Sm = GqSmem<D, GH>;
    constexpr int STAGES = Sm::STAGES;
    constexpr int KS = D / 16;  // k-steps of S
    constexpr int NT = D / 8;   // n-tiles of O
    constexpr int kPage = 256;
    constexpr bool kTwoRows = GH > 8;  // the group fills rows 8..15 of the MMA tile too
    static_assert(GH <= 16, "a group is at most the 16 rows of one MMA tile");
    static_assert(STAGES >= 2 && STAGES % 2 == 0, "ring: an even number of stages");
    static_assert(sizeof(Sm) + 1024 <= kGqSmemLimit, "shared memory");
    extern __shared__ uint8_t gq_smem_raw[];
    Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(gq_smem_raw) + 1023) &
                                    ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&sm.full[i], 1);
            // the four warps of the chunk's team, or all eight when both
            // teams read every chunk
            mbar_init(&sm.empty[i], teams == 2 ? kGqWarps : kGqWarps / 2);
        }
        mbar_init(&sm.cmb, kGqWarps * 32);
        mbar_init(&sm.cfree, kGqWarps * 32);
        sm.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int total_units = __ldg(unit_off + B);
    UnitCursor cur;
    cur.next_off = (B > 1) ? __ldg(unit_off + 1) : 0x7fffffff;

    if (warp == kGqWarps) {
        // ================= producer: TMA boxes of (page, K/V head) slices =================
        if (lane == 0) {
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
        }
        int g = 0;  // ring uses so far
        bool ok = true;
        for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
            const UnitShape us = unit_shape(u, cur, unit_off, page_off, seq_lens, B, Hk, kPage,
                                            max_splits, min_pages);
            const int nchunks = (us.ntok + kGqTok - 1) / kGqTok;
            constexpr int per_page = kPage / kGqTok;
            int z = 0;  // (page, head) slice; -1 reads zeros
            for (int c = 0; c < nchunks; ++c, ++g) {
                if (c % per_page == 0) {
                    const int page = __ldg(page_table + us.pt_base + c / per_page);
                    if (page < 0 || page >= num_pages) {
                        if (lane == 0) record_error(err, FA_DEVERR_BAD_INPUT);
                        z = -1;
                    } else {
                        z = page * (Hk / sub) + us.h / sub;
                    }
                }
                const int slot = g % STAGES;
                if (lane == 0) {
                    if (!mbar_wait(&sm.empty[slot], ((g / STAGES) & 1) ^ 1, err, FA_DEVERR_TIMEOUT,
                                   abort)) {
                        ok = false;
                    } else {
                        const int y = (c % per_page) * kGqTok;
                        mbar_arrive_expect_tx(&sm.full[slot], 2 * Sm::kTile);
#pragma unroll
                        for (int cb = 0; cb < D / 64; ++cb) {
                            tma_load_3d(sm.k[slot] + cb * kGqTok * 128, &tk, &sm.full[slot],
                                        cb * 64, y, z);
                            tma_load_3d(sm.v[slot] + cb * kGqTok * 128, &tv, &sm.full[slot],
                                        cb * 64, y, z);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        // every copy this CTA started must land before it exits
        if (lane == 0)
            for (int i = max(0, g - STAGES); i < g; ++i)
                mbar_wait(&sm.full[i % STAGES], (i / STAGES) & 1, err, FA_DEVERR_TIMEOUT, nullptr);
        __syncwarp();
        return;
    }

    // ================= consumers =================
    const int team = warp >> 2, wt = warp & 3;
    const bool two = teams == 2;
    const int rows = two ? 2 * gr : gr;      // query heads per unit
    const int row_off = two ? team * gr : 0;  // this team's first one
    const int grp = lane >> 2, tig = lane & 3;    // fragment row, column pair
    const int lrow = lane & 7, lmat = lane >> 3;  // ldmatrix row and matrix
    int g = 0, k = 0;                             // ring uses, units done
    bool ok = true;
    for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x, ++k) {
        const UnitShape us = unit_shape(u, cur, unit_off, page_off, seq_lens, B, Hk, kPage,
                                        max_splits, min_pages);
        // the group's query rows as A fragments: a0 / a2 = row grp, columns
        // 16ks + 2tig..+1 / +8; a1 / a3 = the same of row grp + 8 (groups of
        // 16); rows gr..15 are zero
        uint32_t qa[KS][4];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int row = grp + 8 * rr;
            const bool row_in = row < gr;
            const __nv_bfloat16* qr =
                q + (static_cast<int64_t>(us.b) * H + us.h * rows + row_off + (row_in ? row : 0)) *
                        D;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qa[ks][rr] = row_in ? __ldg(reinterpret_cast<const uint32_t*>(qr + ks * 16 + 2 * tig)) : 0u;
                qa[ks][rr + 2] =
                    row_in ? __ldg(reinterpret_cast<const uint32_t*>(qr + ks * 16 + 8 + 2 * tig)) : 0u;
            }
        }
        // rows grp (index 0) and grp + 8 (index 1, groups of 16 only)
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
        const int nchunks = (us.ntok + kGqTok - 1) / kGqTok;
        for (int c = 0; c < nchunks; ++c, ++g) {
            if (!two && (g & 1) != team) continue;
            const int slot = g % STAGES;
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[slot], (g / STAGES) & 1, err,
                                                   FA_DEVERR_TIMEOUT, abort));
            if (!ok) break;
            const uint32_t kb = smem_u32(sm.k[slot]), vb = smem_u32(sm.v[slot]);
            const int t0 = c * kGqTok + 16 * wt;  // the warp's first token in the unit
            // ---- S = Q K^T: n-tile j holds tokens t0 + 8j .. +7
            float s[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    // matrices: column chunks 4kp .. 4kp+3 of token rows 16wt + 8j ..
                    uint32_t b[4];
                    ldsm_x4(b, kb + gq_swz(16 * wt + 8 * j + lrow, 4 * kp + lmat));
                    mma_bf16_16816(s[j], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2],
                                   qa[2 * kp][3], b[0], b[1]);
                    mma_bf16_16816(s[j], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2],
                                   qa[2 * kp + 1][3], b[2], b[3]);
                }
            }
            // ---- online softmax of rows grp (and grp + 8) over this warp's 16 tokens
            const bool partial = t0 + 16 > us.ntok;
            uint32_t pa[4];  // P as the A operand, as qa
#pragma unroll
            for (int rr = 0; rr < (kTwoRows ? 2 : 1); ++rr) {
                float sv[4];
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float x = s[j][2 * rr + e] * scale_log2;
                        sv[2 * j + e] =
                            (partial && t0 + 8 * j + 2 * tig + e >= us.ntok) ? -INFINITY : x;
                    }
                float mb = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
                const float mn = fmaxf(m[rr], mb);
                const float mu = (mn == -INFINITY) ? 0.f : mn;  // no finite score yet
                const float alpha = ex2_approx(m[rr] - mu);      // m = -inf -> 0
                l[rr] *= alpha;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    acc[n][2 * rr] *= alpha;
                    acc[n][2 * rr + 1] *= alpha;
                }
                float pv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) pv[i] = ex2_approx(sv[i] - mu);  // -inf -> 0
                l[rr] += (pv[0] + pv[1]) + (pv[2] + pv[3]);
                m[rr] = mn;
                // tokens 2tig..+1 of n-tile 0 (k columns 0-7) and n-tile 1 (8-15)
                pa[rr] = pack_bf16x2(pv[0], pv[1]);
                pa[rr + 2] = pack_bf16x2(pv[2], pv[3]);
            }
            if constexpr (!kTwoRows) pa[1] = pa[3] = 0u;
            // V rows past the unit's tokens may hold anything (0 * NaN): zero
            // their halves of the B fragments
            uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
            if (partial) {
                const int tt = t0 + 2 * tig;
                mlo = (tt < us.ntok ? 0x0000ffffu : 0u) | (tt + 1 < us.ntok ? 0xffff0000u : 0u);
                mhi = (tt + 8 < us.ntok ? 0x0000ffffu : 0u) | (tt + 9 < us.ntok ? 0xffff0000u : 0u);
            }
            // ---- O += P V: matrices (tokens 0-7 | 8-15) x (column chunk 2np | 2np+1)
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b[4];
                ldsm_x4_trans(b, vb + gq_swz(16 * wt + 8 * (lmat & 1) + lrow, 2 * np + (lmat >> 1)));
                mma_bf16_16816(acc[2 * np], pa[0], pa[1], pa[2], pa[3], b[0] & mlo, b[1] & mhi);
                mma_bf16_16816(acc[2 * np + 1], pa[0], pa[1], pa[2], pa[3], b[2] & mlo,
                               b[3] & mhi);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
        if (!ok) break;
        // ---- merge the 8 warps' states of this unit through the one buffer,
        // once every consumer has read the previous unit's merge out of it
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 1);
            l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 2);
        }
        if (k > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.cfree, (k - 1) & 1, err, FA_DEVERR_TIMEOUT,
                                                   abort));
            if (!ok) break;
        }
#pragma unroll
        for (int rr = 0; rr < (kTwoRows ? 2 : 1); ++rr) {
            const int row = grp + 8 * rr;
            if (row < gr) {
                if (tig == 0) {
                    sm.cm[row][warp] = m[rr];
                    sm.cl[row][warp] = l[rr];
                }
#pragma unroll
                for (int n = 0; n < NT; ++n)
                    *reinterpret_cast<float2*>(&sm.co[row][warp][n * 8 + 2 * tig]) =
                        make_float2(acc[n][2 * rr], acc[n][2 * rr + 1]);
            }
        }
        mbar_arrive(&sm.cmb);
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.cmb, k & 1, err, FA_DEVERR_TIMEOUT, abort));
        if (!ok) break;
        for (int idx = threadIdx.x; idx < rows * D; idx += kGqWarps * 32) {
            const int ha = idx / D, x = idx - ha * D;  // the unit's query head, column
            // the warps holding that head's states: its team's four, or all
            const int tt = two ? ha / gr : 0;
            const int hi = ha - tt * gr;
            float M = -INFINITY, L = 0.f, o = 0.f;
            auto combine = [&](int w0, auto nw_c) {
                constexpr int NW = decltype(nw_c)::value;
#pragma unroll
                for (int w = 0; w < NW; ++w) M = fmaxf(M, sm.cm[hi][w0 + w]);
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    const float mw = sm.cm[hi][w0 + w];
                    const float wgt = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
                    L += wgt * sm.cl[hi][w0 + w];
                    o += wgt * sm.co[hi][w0 + w][x];
                }
            };
            if (two) combine(4 * tt, std::integral_constant<int, kGqWarps / 2>{});
            else combine(0, std::integral_constant<int, kGqWarps>{});
            const int64_t pu = static_cast<int64_t>(u) * rows + ha;
            part_o[pu * D + x] = o / L;
            if (x == 0) part_lse[pu] = M + __log2f(L);
        }
        mbar_arrive(&sm.cfree);
    }
}

// One warp per (sequence, query head).  Sequence b's partials start at
// unit_off[b] * GH and are split-major with H per split.
template <int D>
__global__ void __launch_bounds__(128)
    fa_decode_merge_kernel(const int32_t* __restrict__ seq_lens, int B, int H, int GH,
                           int page_size, int max_splits, int min_pages,
                           const int32_t* __restrict__ unit_off,
                           const float* __restrict__ part_lse, const float* __restrict__ part_o,
                           __nv_bfloat16* __restrict__ o) {
    constexpr int PER = D / 32;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= B * H) return;
    const int b = gw / H, h = gw % H;
    int len = __ldg(seq_lens + b);
    if (len < 0) len = 0;
    const int np = (len + page_size - 1) / page_size;
    int ns, cp;
    split_shape(np, max_splits, min_pages, ns, cp);
    const int base = __ldg(unit_off + b) * GH;
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, part_lse[base + s * H + h]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f, acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    for (int s = 0; s < ns; ++s) {
        const int unit = base + s * H + h;
        const float w = ex2_approx(part_lse[unit] - M);
        L += w;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, part_o[static_cast<int64_t>(unit) * D + lane * PER + i], acc[i]);
    }
    const float inv = ns > 0 ? 1.f / L : 0.f;
    __nv_bfloat16* dst = o + (static_cast<int64_t>(b) * H + h) * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2) {
        const uint32_t pk = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
        *reinterpret_cast<uint32_t*>(dst + i) = pk;
    }
}

// Grid-stride over the pages of all sequences; copies each page's valid
// tokens, all heads, into the contiguous output rows.
template <int D>
__global__ void __launch_bounds__(256)
    fa_gather_kernel(const __nv_bfloat16* __restrict__ pages,
                     const int32_t* __restrict__ page_table,
                     const int32_t* __restrict__ seq_lens, int B, int H, int page_size,
                     const int32_t* __restrict__ page_off, const int32_t* __restrict__ tok_off,
                     __nv_bfloat16* __restrict__ out) {
    constexpr int V = D / 8;  // 16-byte vectors per row
    const int total_pages = __ldg(page_off + B);
    for (int g = blockIdx.x; g < total_pages; g += gridDim.x) {
        const int b = find_owner(page_off, B, g);
        const int i = g - __ldg(page_off + b);
        int len = __ldg(seq_lens + b);
        if (len < 0) len = 0;
        const int t0 = i * page_size;
        const int cnt = min(page_size, len - t0);
        const int page = __ldg(page_table + g);
        const int64_t row0 = __ldg(tok_off + b) + t0;
        const int work = H * cnt * V;
        for (int x = threadIdx.x; x < work; x += blockDim.x) {
            const int vec = x % V;
            const int slot = (x / V) % cnt;
            const int hh = x / (V * cnt);
            const uint4 val = *reinterpret_cast<const uint4*>(
                pages + ((static_cast<int64_t>(page) * H + hh) * page_size + slot) * D + vec * 8);
            *reinterpret_cast<uint4*>(out + ((row0 + slot) * H + hh) * D + vec * 8) = val;
        }
    }
}

// Appends the new K and V rows of every sequence to the paged cache: new row
// g of sequence b (cu_new[b] <= g < cu_new[b+1]) is the sequence's token
// pos = seq_lens[b] - n_b + (g - cu_new[b]) (seq_lens counts the tokens after
// the append) and goes to slot pos % page_size of page
// page_table[page_off[b] + pos / page_size].  Grid-stride over 16-byte words.
// A sequence with more new rows than tokens, or a page index outside the
// pool, is skipped and reported; no write leaves the pool.
template <int D>
__global__ void __launch_bounds__(256)
    fa_append_kernel(const __nv_bfloat16* __restrict__ k_new,
                     const __nv_bfloat16* __restrict__ v_new, const int32_t* __restrict__ cu_new,
                     __nv_bfloat16* __restrict__ k_pages, __nv_bfloat16* __restrict__ v_pages,
                     const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
                     const int32_t* __restrict__ page_off, int B, int Hk, int total_new,
                     int page_size, int num_pages, unsigned int* err) {
    constexpr int V = D / 8;  // 16-byte words per row
    const int64_t words = static_cast<int64_t>(total_new) * Hk * V;
    for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < words;
         x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int vec = static_cast<int>(x % V);
        const int hh = static_cast<int>((x / V) % Hk);
        const int g = static_cast<int>(x / (static_cast<int64_t>(V) * Hk));
        const int b = find_owner(cu_new, B, g);
        const int n = __ldg(cu_new + b + 1) - __ldg(cu_new + b);
        const int len = __ldg(seq_lens + b);
        if (n > len || n < 0) {
            if (vec == 0 && hh == 0) record_error(err, FA_DEVERR_BAD_INPUT);
            continue;
        }
        const int pos = len - n + (g - __ldg(cu_new + b));
        const int page = __ldg(page_table + __ldg(page_off + b) + pos / page_size);
        if (page < 0 || page >= num_pages) {
            record_error(err, FA_DEVERR_BAD_INPUT);
            continue;
        }
        const int64_t src = (static_cast<int64_t>(g) * Hk + hh) * D + vec * 8;
        const int64_t dst =
            ((static_cast<int64_t>(page) * Hk + hh) * page_size + pos % page_size) * D + vec * 8;
        *reinterpret_cast<uint4*>(k_pages + dst) = *reinterpret_cast<const uint4*>(k_new + src);
        *reinterpret_cast<uint4*>(v_pages + dst) = *reinterpret_cast<const uint4*>(v_new + src);
    }
}

// gr query heads per team (gr <= GH, the kernel's capacity; GH == 1 is the
// multi-head kernel), teams sub-groups per unit, sub units per K/V head (a
// group of gr * teams * sub)
template <int D, int GH>
int launch_decode_impl(const void* q, const void* k_pages, const void* v_pages,
                       const CUtensorMap* tk, const CUtensorMap* tv, const int32_t* page_table,
                       const int32_t* seq_lens, void* o, int B, int H, int num_pages,
                       int page_size, int max_splits, void* workspace, unsigned int* err,
                       int num_sms, cudaStream_t stream, int gr, int sub, int teams = 1) {
    const int rows = gr * teams;  // query heads per unit
    const int Hk = H / rows;      // units per split
    // pages a split covers at least: with few units per split (few K/V heads),
    // larger splits keep the partials and per-unit merges down
    const int min_pages = Hk >= kDecodeManyUnits ? kDecodeChunkPages : kDecodeChunkPagesFew;
    const WorkspaceLayout L = layout_of(B, H, D, max_splits);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* page_off = reinterpret_cast<int32_t*>(ws);
    int32_t* tok_off = page_off + (B + 1);
    int32_t* unit_off = tok_off + (B + 1);
    float* part_lse = reinterpret_cast<float*>(ws + L.lse_off);
    float* part_o = reinterpret_cast<float*>(ws + L.o_off);
    // units are (split, K/V head) pairs
    fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, B, Hk, page_size, max_splits,
                                                          min_pages, page_off, tok_off, unit_off,
                                                          err);
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    if constexpr (GH == 1) {
        auto split = fa_decode_split_kernel<D>;
        const size_t smem = sizeof(DecSmem<D>) + 128;
        if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return FA_ERR_CUDA;
        // a persistent grid of the CTAs that are resident at once
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, split, kDecThreads, smem) !=
                cudaSuccess ||
            occ < 1)
            return FA_ERR_CUDA;
        split<<<num_sms * occ, kDecThreads, smem, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_pages),
            static_cast<const __nv_bfloat16*>(v_pages), page_table, seq_lens, B, H, num_pages,
            page_size, max_splits, min_pages, page_off, unit_off, part_lse, part_o, scale_log2,
            err);
    } else {
        if (!tk || !tv) return FA_ERR_NULL;
        auto split = fa_decode_gqa_kernel<D, GH>;
        const size_t smem = sizeof(GqSmem<D, GH>) + 1024;
        if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return FA_ERR_CUDA;
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, split, kGqThreads, smem) !=
                cudaSuccess ||
            occ < 1)
            return FA_ERR_CUDA;
        split<<<num_sms * occ, kGqThreads, smem, stream>>>(
            *tk, *tv, static_cast<const __nv_bfloat16*>(q), page_table, seq_lens, B, H, Hk, gr, sub,
            teams, num_pages, max_splits, min_pages, page_off, unit_off, part_lse, part_o,
            scale_log2, err);
    }
    const int warps = B * H;
    fa_decode_merge_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(
        seq_lens, B, H, rows, page_size, max_splits, min_pages, unit_off, part_lse, part_o,
        static_cast<__nv_bfloat16*>(o));
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
int launch_gather_impl(const void* pages, const int32_t* page_table, const int32_t* seq_lens,
                       void* out, int B, int H, int page_size, void* workspace, unsigned int* err,
                       int num_sms, cudaStream_t stream) {
    int32_t* page_off = static_cast<int32_t*>(workspace);
    int32_t* tok_off = page_off + (B + 1);
    int32_t* unit_off = tok_off + (B + 1);
    fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, B, H, page_size, 1, 1, page_off,
                                                          tok_off, unit_off, err);
    fa_gather_kernel<D><<<num_sms * 8, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(pages), page_table, seq_lens, B, H, page_size,
        page_off, tok_off, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
int launch_append_impl(const void* k_new, const void* v_new, const int32_t* cu_new, void* k_pages,
                       void* v_pages, const int32_t* page_table, const int32_t* seq_lens, int B,
                       int Hk, int total_new, int page_size, int num_pages, void* workspace,
                       unsigned int* err, int num_sms, cudaStream_t stream) {
    int32_t* page_off = static_cast<int32_t*>(workspace);
    int32_t* tok_off = page_off + (B + 1);
    int32_t* unit_off = tok_off + (B + 1);
    fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, B, Hk, page_size, 1, 1, page_off,
                                                          tok_off, unit_off, err);
    fa_append_kernel<D><<<num_sms * 8, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), cu_new,
        static_cast<__nv_bfloat16*>(k_pages), static_cast<__nv_bfloat16*>(v_pages), page_table,
        seq_lens, page_off, B, Hk, total_new, page_size, num_pages, err);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

int launch_append(const void* k_new, const void* v_new, const int32_t* cu_new, void* k_pages,
                  void* v_pages, const int32_t* page_table, const int32_t* seq_lens, int B,
                  int Hk, int total_new, int d, int page_size, int num_pages, void* workspace,
                  unsigned int* err, int num_sms, cudaStream_t stream) {
    if (d == 128)
        return launch_append_impl<128>(k_new, v_new, cu_new, k_pages, v_pages, page_table,
                                       seq_lens, B, Hk, total_new, page_size, num_pages,
                                       workspace, err, num_sms, stream);
    if (d == 64)
        return launch_append_impl<64>(k_new, v_new, cu_new, k_pages, v_pages, page_table,
                                      seq_lens, B, Hk, total_new, page_size, num_pages,
                                      workspace, err, num_sms, stream);
    return FA_ERR_UNSUPPORTED;
}

size_t decode_workspace_bytes(int B, int H, int d, int max_splits) {
    return layout_of(B, H, d, max_splits).total;
}

int launch_decode_pack(const int32_t* block_table, int max_pages, const int32_t* seq_lens, int B,
                       int page_size, int32_t* packed, int32_t* lens, unsigned int* err,
                       cudaStream_t stream) {
    fa_decode_pack_kernel<<<1, kPlanThreads, 0, stream>>>(block_table, max_pages, seq_lens, B,
                                                          page_size, packed, lens, err);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

namespace {
template <int D>
int launch_decode_d(const void* q, const void* k_pages, const void* v_pages,
                    const CUtensorMap* tk, const CUtensorMap* tv, const int32_t* page_table,
                    const int32_t* seq_lens, void* o, int B, int H, int Hk, int num_pages,
                    int page_size, int max_splits, void* workspace, unsigned int* err,
                    int num_sms, cudaStream_t stream) {
    // a group of G query heads per K/V head is cut into sub sub-groups of
    // gr = G / sub heads, sub the fewest that leaves gr <= 16; an even number
    // of sub-groups runs as pairs, one unit per pair (both read each chunk)
    const int G = H / Hk;
    int sub = (G + 15) / 16;
    while (G % sub != 0) ++sub;
    const int gr = G / sub;
    const int teams = (sub % 2 == 0) ? 2 : 1;
    if (G == 1)
        return launch_decode_impl<D, 1>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, B,
                                        H, num_pages, page_size, max_splits, workspace, err,
                                        num_sms, stream, 1, 1);
#define FA_DECODE_GH(GH)                                                                        \
    if (gr <= GH)                                                                               \
        return launch_decode_impl<D, GH>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, \
                                         B, H, num_pages, page_size, max_splits, workspace,    \
                                         err, num_sms, stream, gr, sub / teams, teams);
    FA_DECODE_GH(2)
    FA_DECODE_GH(4)
    FA_DECODE_GH(8)
    FA_DECODE_GH(16)
#undef FA_DECODE_GH
    return FA_ERR_UNSUPPORTED;
}
}  // namespace

bool decode_group_supported(int H, int Hk) { return Hk >= 1 && H % Hk == 0; }

int launch_decode(const void* q, const void* k_pages, const void* v_pages,
                  const CUtensorMap* tk, const CUtensorMap* tv, const int32_t* page_table,
                  const int32_t* seq_lens, void* o, int B, int H, int Hk, int num_pages, int d,
                  int page_size, int max_splits, void* workspace, unsigned int* err, int num_sms,
                  cudaStream_t stream) {
    if (!decode_group_supported(H, Hk)) return FA_ERR_UNSUPPORTED;
    if (d == 128)
        return launch_decode_d<128>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, B, H,
                                    Hk, num_pages, page_size, max_splits, workspace, err, num_sms,
                                    stream);
    if (d == 64)
        return launch_decode_d<64>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, B, H, Hk,
                                   num_pages, page_size, max_splits, workspace, err, num_sms,
                                   stream);
    return FA_ERR_UNSUPPORTED;
}

int launch_gather(const void* pages, const int32_t* page_table, const int32_t* seq_lens,
                  void* out, int B, int H, int d, int page_size, void* workspace,
                  unsigned int* err, int num_sms, cudaStream_t stream) {
    if (d == 128)
        return launch_gather_impl<128>(pages, page_table, seq_lens, out, B, H, page_size,
                                       workspace, err, num_sms, stream);
    if (d == 64)
        return launch_gather_impl<64>(pages, page_table, seq_lens, out, B, H, page_size,
                                      workspace, err, num_sms, stream);
    return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
