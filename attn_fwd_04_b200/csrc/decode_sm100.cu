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
// Grouped query heads (several per K/V head) take the same three steps with
// a kernel of their own (below): its dot products run on the tensor cores,
// and with one or two unit heads per sequence (multi-query attention) the
// plan splits the chunk stream of all sequences evenly over the CTAs
// instead of cutting each sequence into splits of its own.
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
// ---------------------------------------------------------------------------
// Balanced partition of the grouped decode.  Slab s = b * Hk + h (sequence
// b, unit head h) holds nc_b = ceil(len_b / 64) chunks of 64 tokens; the
// slabs lie end to end in one stream of W = Hk * sum_b nc_b chunks (slab
// (b, h) starts at Hk * C_b + h * nc_b, C_b the chunks of the sequences
// before b), and CTA i of G takes chunks [i W / G, (i + 1) W / G).  A piece
// is what one CTA takes of one slab; slab s's pieces are its CTAs in order,
// and its partial results are rows slab_base[s] + j, j the piece.  Every
// CTA then has the same work to within one chunk, and a short sequence
// costs one piece rather than a split of its own.  With fewer chunks than
// CTAs only the first W CTAs take part (G below is min(CTAs, W)), so that
// every range is non-empty and every CTA between a slab's first and last
// holds a piece of it.
// ---------------------------------------------------------------------------
constexpr int kSkTok = 64;  // tokens per chunk of the stream

__host__ __device__ inline int64_t sk_bnd(int i, int64_t W, int G) {
    return static_cast<int64_t>(i) * W / G;
}
// the CTA whose range holds stream position x (0 < G <= W)
__host__ __device__ inline int sk_cta_of(int64_t x, int64_t W, int G) {
    return static_cast<int>(((x + 1) * G - 1) / W);
}
// the CTAs that take part: min(grid, W)
__host__ __device__ inline int sk_ctas(int grid, int64_t W) {
    return static_cast<int>(W < grid ? W : grid);
}

struct SkLayout {
    size_t page_off, cnk_off, slab_base, first_slab, lse_off, o_off, total;
};

// Workspace of the grouped decode: page and chunk prefixes per sequence,
// the first partial row of each slab, each CTA's first slab, then the
// partial log-sum-exps and outputs of at most B * Hk + G pieces of rows
// query heads each.
__host__ __device__ inline SkLayout sk_layout_of(int B, int Hk, int rows, int d, int G) {
    SkLayout L;
    size_t at = 0;
    L.page_off = at;
    at += sizeof(int32_t) * (static_cast<size_t>(B) + 1);
    L.cnk_off = at;
    at += sizeof(int32_t) * (static_cast<size_t>(B) + 1);
    L.slab_base = at;
    at += sizeof(int32_t) * (static_cast<size_t>(B) * Hk + 1);
    L.first_slab = at;
    at += sizeof(int32_t) * static_cast<size_t>(G);
    const size_t prow = (static_cast<size_t>(B) * Hk + G) * rows;
    L.lse_off = align256(at);
    L.o_off = L.lse_off + align256(sizeof(float) * prow);
    L.total = L.o_off + sizeof(float) * prow * d;
    return L;
}

__global__ void __launch_bounds__(kPlanThreads)
    fa_decode_sk_plan_kernel(const int32_t* __restrict__ seq_lens, int B, int Hk, int G,
                             int32_t* page_off, int32_t* cnk_off, int32_t* slab_base,
                             int32_t* first_slab, unsigned int* err) {
    __shared__ int sh[32];
    int carry_p = 0, carry_c = 0;
    if (threadIdx.x == 0) {
        page_off[0] = 0;
        cnk_off[0] = 0;
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
        int tp, tc;
        const int ip = block_incl_scan((len + 255) / 256, sh, tp);
        const int ic = block_incl_scan((len + kSkTok - 1) / kSkTok, sh, tc);
        if (i < B) {
            page_off[i + 1] = carry_p + ip;
            cnk_off[i + 1] = carry_c + ic;
        }
        carry_p += tp;
        carry_c += tc;
    }
    __syncthreads();  // cnk_off is read back below
    const int64_t W = static_cast<int64_t>(Hk) * carry_c;
    G = sk_ctas(G, W);
    const int slabs = B * Hk;
    int carry_s = 0;
    if (threadIdx.x == 0) slab_base[0] = 0;
    for (int base = 0; base < slabs; base += kPlanThreads) {
        const int sl = base + threadIdx.x;
        int pieces = 0;
        if (sl < slabs) {
            const int b = sl / Hk, h = sl - b * Hk;
            const int c0 = cnk_off[b], nc = cnk_off[b + 1] - c0;
            if (nc > 0) {
                const int64_t start = static_cast<int64_t>(Hk) * c0 + static_cast<int64_t>(h) * nc;
                const int lo = sk_cta_of(start, W, G), hi = sk_cta_of(start + nc - 1, W, G);
                pieces = hi - lo + 1;
                // the CTAs whose range starts inside this slab begin with it
                for (int c = lo; c <= hi; ++c)
                    if (sk_bnd(c, W, G) >= start) first_slab[c] = sl;
            }
        }
        int tot;
        const int inc = block_incl_scan(pieces, sh, tot);
        if (sl < slabs) slab_base[sl + 1] = carry_s + inc;
        carry_s += tot;
    }
}

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
                           float* __restrict__ part_o, float scale_log2, unsigned int* err,
                           uint64_t wait_ns, int withhold) {
    // wait_ns, withhold: the failure-detection check only (0 in every other
    // call): the bound of every wait (0: FA_WAIT_TIMEOUT_NS), and 1 + the ring
    // use at which the producer stops issuing copies (0: none)
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
    const uint64_t wlim = wait_ns ? wait_ns : FA_WAIT_TIMEOUT_NS;
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
                if (g + 1 == withhold) {  // failure-detection check: no more copies
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    if (!mbar_wait(&sm.empty[slot], ((g / kDecStages) & 1) ^ 1, err,
                                   FA_DEVERR_TIMEOUT, abort, wlim)) {
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
                          nullptr, wlim);
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
                               abort, wlim)) {
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
            if (!mbar_wait(&sm.cmb[par], (k >> 1) & 1, err, FA_DEVERR_TIMEOUT, abort, wlim)) {
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
// Grouped query heads (groups of 2 or more; see below for the sizes).  The
// GH query heads of a unit are the rows of a 16-row MMA tile (rows GH..15 are
// zero), so each staged K/V byte serves all of them and the dot products run
// as small matrix products on the tensor cores (warp-level m16n8k16; a
// tcgen05 form, S^T = K Q^T with the chunk as M, measured slower: with 32
// heads as N its operand reads outrun shared memory).  K/V chunks of 64
// tokens arrive by TMA in the 128-byte-swizzled layout, so the ldmatrix reads
// of 8 token rows at one column fall in 8 distinct bank groups.  A warp takes
// WT consecutive tokens of a chunk, so 64 / WT warps cover a chunk for one
// set of rows:
//   S  = Q_g K^T   WT/8 8-token n-tiles over D/16 k-steps (fp32)
//   online softmax per query row (rows lane / 4 and, for groups of 16,
//   lane / 4 + 8; the 4 lanes of a quad share them), base 2 with
//   scale * log2(e) applied to S
//   O += P V       P from S's accumulators as the A operand, V through
//                  ldmatrix.trans, D/8 n-tiles over WT/16 k-steps
// The warps covering one chunk for one set of rows form a crew, and two
// crews per set of rows take the chunks in turn.
// Groups larger than 16 (multi-query attention with many heads) are cut into
// equal sub-groups of gr <= 16 query heads (GH, the template, is the capacity
// of the registers and merge slots).  An even number of sub-groups is paired:
// a unit then holds two sub-groups of the same K/V head (warps 0-3 the first
// one's rows, warps 4-7 the second's, each half covering every chunk), so a
// staged chunk serves 2 gr query heads and is read from memory once for both,
// and a warp takes 32 tokens (its softmax row bookkeeping -- max shuffles,
// the rescale of the D/4 accumulators of a row pair -- is paid once per 32
// tokens, not 16).  Otherwise a unit holds one sub-group and a warp 16
// tokens.  Hk counts the unit heads per sequence (H / rows) and sub the unit
// heads per K/V head: a unit head h reads K/V head h / sub.
// At the end of a unit the 8 warps' (m, l, O) are merged in two rounds
// through 4 slots (crew 1 into crew 0, then the slots of each set of rows),
// which leaves room for 6 ring stages.  The producer warp walks the units --
// split units taken in turn, or the pieces of the evenly split chunk stream
// for one or two unit heads (see launch_decode_gqa) -- and hands each one's
// shape to the consumers.
// ---------------------------------------------------------------------------
constexpr int kGqTok = 64;          // tokens per chunk
constexpr int kGqWarps = 8;         // consumer warps
constexpr int kGqThreads = (kGqWarps + 1) * 32;
constexpr int kGqSmemLimit = 232448;  // opt-in shared memory per block

template <int D, int GH, int WT>
struct GqSmem {
    static constexpr int kTile = kGqTok * D * 2;   // one of K, V per stage
    // the merge goes through one slot per warp of a crew and set of rows
    // (4 for both shapes: 2 teams x 2 warps, or 1 team x 4 warps); a slot's
    // partial O rows are kCoStride floats apart, so the 8 rows of one float2
    // store fall on 8 bank quads that cover every bank twice (2 wavefronts,
    // the least for 64 words) and the combine's float4 reads stay aligned
    static constexpr int kSlots = 4;
    static constexpr int kCoStride = D + 4;
    static constexpr int kCo = kSlots * GH * kCoStride * 4;
    static constexpr int kMisc = 2 * GH * kSlots * 4 + 256;  // cm, cl, barriers
    static constexpr int kFit = (kGqSmemLimit - 1024 - kCo - kMisc) / (2 * kTile);
    // chunk g goes to crew g % 2 and stage g % STAGES; an even count keeps
    // each stage with one crew, which then sees every phase of its barriers
    // in order (with an odd count a crew could wait on a stage two phases
    // ahead of it, and a parity wait cannot tell those phases apart)
    static constexpr int STAGES = (kFit < 6 ? kFit : 6) & ~1;
    alignas(1024) uint8_t k[STAGES][kTile];
    alignas(1024) uint8_t v[STAGES][kTile];
    // per-slot partial state of the unit being merged; c1: crew 1 has
    // written its states, cmb: crew 0 has written the pairwise merges,
    // cfree: every consumer has read the merged unit
    float co[kSlots][GH][kCoStride];
    float cm[GH][kSlots], cl[GH][kSlots];
    // the producer hands each unit's shape to the consumers through two
    // slots (unit k in slot k % 2): ud_full when written, ud_empty when
    // every consumer has read it
    int ud[2][8];
    uint64_t full[STAGES], empty[STAGES], c1, cmb, cfree, ud_full[2], ud_empty[2];
    int abort;
};

// Byte offset of (token t, 16-byte column chunk c) in a staged tile: D/64
// TMA boxes of 64 rows x 128 bytes, chunk index XOR (row % 8) inside a box.
__device__ __forceinline__ uint32_t gq_swz(int t, int c) {
    return static_cast<uint32_t>((c >> 3) * (kGqTok * 128) + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

template <int D, int GH, int WT>
__global__ void __launch_bounds__(kGqThreads, 1)
    fa_decode_gqa_kernel(const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv,
                         const __nv_bfloat16* __restrict__ q,
                         const int32_t* __restrict__ page_table,
                         const int32_t* __restrict__ seq_lens, int B, int H, int Hk, int gr, int sub,
                         int num_pages, int balanced, const int32_t* __restrict__ page_off,
                         const int32_t* __restrict__ cnk_off,
                         const int32_t* __restrict__ slab_base,
                         const int32_t* __restrict__ first_slab,
                         const int32_t* __restrict__ unit_off, int max_splits, int min_pages,
                         float* __restrict__ part_lse, float* __restrict__ part_o,
                         float scale_log2, unsigned int* err) {
    using Sm = GqSmem<D, GH, WT>;
    constexpr int STAGES = Sm::STAGES;
    constexpr int KS = D / 16;  // k-steps of S
    constexpr int NT = D / 8;   // n-tiles of O
    constexpr int NJ = WT / 8;  // n-tiles of S (8 tokens each)
    constexpr int KP = WT / 16; // k-steps of P V (16 tokens each)
    constexpr int kCrewWarps = kGqTok / WT;  // warps covering one chunk for one set of rows
    // 32 tokens per warp when a unit pairs two sub-groups, 16 when it holds
    // one; either way two crews per set of rows take the chunks in turn
    constexpr int kTeams = WT / 16;
    constexpr bool kTwo = kTeams == 2;
    static_assert(kTeams * kCrewWarps * 2 == kGqWarps && kTeams * kCrewWarps == Sm::kSlots,
                  "two crews per set of rows, one merge slot per warp of a crew");
    constexpr int kPage = 256;
    constexpr bool kTwoRows = GH > 8;  // the group fills rows 8..15 of the MMA tile too
    static_assert(GH <= 16, "a group is at most the 16 rows of one MMA tile");
    static_assert(WT == 16 || WT == 32, "16 or 32 tokens per warp");
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
            // the warps that read the chunk: one crew per set of rows
            mbar_init(&sm.empty[i], kTeams * kCrewWarps);
        }
        mbar_init(&sm.c1, kGqWarps / 2 * 32);
        mbar_init(&sm.cmb, kGqWarps / 2 * 32);
        mbar_init(&sm.cfree, kGqWarps * 32);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.ud_full[i], 1);
            mbar_init(&sm.ud_empty[i], kGqWarps * 32);
        }
        sm.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == kGqWarps) {
        // ================= producer: TMA boxes of (page, K/V head) slices =================
        if (lane == 0) {
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
        }
        int g = 0;  // ring uses so far
        bool ok = true;
        // piece k's descriptor for the consumers (b, unit head, tokens,
        // first partial row; tokens < 0 ends the list), once they have read
        // piece k - 2's
        auto hand_over = [&](int k, int b, int h, int ntok, int prow) {
            if (lane == 0) {
                if (k >= 2 && !mbar_wait(&sm.ud_empty[k & 1], ((k - 2) >> 1) & 1, err,
                                         FA_DEVERR_TIMEOUT, abort)) {
                    ok = false;
                } else {
                    int* d = sm.ud[k & 1];
                    d[0] = b;
                    d[1] = h;
                    d[2] = ntok;
                    d[3] = prow;
                    mbar_arrive(&sm.ud_full[k & 1]);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        };
        constexpr int per_page = kPage / kGqTok;
        // chunks c0 .. c1 - 1 of sequence b, unit head h, into the ring
        auto stream_piece = [&](int b, int h, int c0, int c1) {
            const int pt_base = __ldg(page_off + b);
            int z = 0;  // (page, head) slice; -1 reads zeros
            for (int c = c0; c < c1; ++c, ++g) {
                if (c == c0 || c % per_page == 0) {
                    const int page = __ldg(page_table + pt_base + c / per_page);
                    if (page < 0 || page >= num_pages) {
                        if (lane == 0) record_error(err, FA_DEVERR_BAD_INPUT);
                        z = -1;
                    } else {
                        z = page * (Hk / sub) + h / sub;
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
                        for (int cb2 = 0; cb2 < D / 64; ++cb2) {
                            tma_load_3d(sm.k[slot] + cb2 * kGqTok * 128, &tk, &sm.full[slot],
                                        cb2 * 64, y, z);
                            tma_load_3d(sm.v[slot] + cb2 * kGqTok * 128, &tv, &sm.full[slot],
                                        cb2 * 64, y, z);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        };
        int k = 0;  // pieces handed over
        if (balanced) {
            const int64_t W = static_cast<int64_t>(Hk) * __ldg(cnk_off + B);
            const int G = sk_ctas(static_cast<int>(gridDim.x), W);
            const bool mine = static_cast<int>(blockIdx.x) < G;  // W == 0: nobody's
            int64_t x = mine ? sk_bnd(blockIdx.x, W, G) : 0;
            const int64_t x1 = mine ? sk_bnd(blockIdx.x + 1, W, G) : 0;
            int sl = x < x1 ? __ldg(first_slab + blockIdx.x) : 0;
            while (ok && x < x1) {
                // the plan puts x inside slab sl or a later one; anything else
                // is a broken plan, reported, and the rest of the range skipped
                if (sl < 0 || sl >= B * Hk) {
                    if (lane == 0) record_error(err, FA_DEVERR_BAD_INPUT);
                    break;
                }
                const int b = sl / Hk, h = sl - b * Hk;
                const int cb = __ldg(cnk_off + b), nc = __ldg(cnk_off + b + 1) - cb;
                const int64_t start =
                    static_cast<int64_t>(Hk) * cb + static_cast<int64_t>(h) * nc;
                if (nc == 0 || x >= start + nc) {  // an empty sequence's slab, or one behind x
                    ++sl;
                    continue;
                }
                if (x < start) {
                    if (lane == 0) record_error(err, FA_DEVERR_BAD_INPUT);
                    break;
                }
                const int c0 = static_cast<int>(x - start);
                const int c1 = static_cast<int>(min(static_cast<int64_t>(nc), x1 - start));
                int len = __ldg(seq_lens + b);
                if (len < 0) len = 0;
                const int prow = __ldg(slab_base + sl) + (blockIdx.x - sk_cta_of(start, W, G));
                hand_over(k++, b, h, min(len, c1 * kGqTok) - c0 * kGqTok, prow);
                if (!ok) break;
                stream_piece(b, h, c0, c1);
                x = start + c1;
                ++sl;
            }
        } else {
            // split units, u = blockIdx.x, + gridDim.x, ...: the CTAs at work
            // at one time read neighbouring units, i.e. the heads of the same
            // pages
            UnitCursor cur;
            cur.next_off = (B > 1) ? __ldg(unit_off + 1) : 0x7fffffff;
            const int total_units = __ldg(unit_off + B);
            for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
                const UnitShape us = unit_shape(u, cur, unit_off, page_off, seq_lens, B, Hk,
                                                kPage, max_splits, min_pages);
                hand_over(k++, us.b, us.h, us.ntok, u);
                if (!ok) break;
                const int c0 = us.tok0 / kGqTok;
                stream_piece(us.b, us.h, c0, c0 + (us.ntok + kGqTok - 1) / kGqTok);
            }
        }
        if (ok) hand_over(k, 0, 0, -1, 0);
        // every copy this CTA started must land before it exits
        if (lane == 0)
            for (int i = max(0, g - STAGES); i < g; ++i)
                mbar_wait(&sm.full[i % STAGES], (i / STAGES) & 1, err, FA_DEVERR_TIMEOUT, nullptr);
        __syncwarp();
        return;
    }

    // ================= consumers =================
    const int team = kTwo ? warp >> 2 : 0;          // the set of rows: sub-group
    const int crew = (warp / kCrewWarps) & 1;       // takes chunks g % 2 == crew
    const int wc = warp % kCrewWarps;               // the warp's place in its crew
    const int tbase = WT * wc;                      // its first token in a chunk
    const int mslot = team * kCrewWarps + wc;       // its merge slot
    const int rows = kTwo ? 2 * gr : gr;      // query heads per unit
    const int row_off = kTwo ? team * gr : 0;  // this team's first one
    const int grp = lane >> 2, tig = lane & 3;    // fragment row, column pair
    const int lrow = lane & 7, lmat = lane >> 3;  // ldmatrix row and matrix
    int g = 0, k = 0;                             // ring uses, units done
    bool ok = true;
    // the group's query rows as A fragments: a0 / a2 = row grp, columns
    // 16ks + 2tig..+1 / +8; a1 / a3 = the same of row grp + 8 (groups of
    // 16); rows gr..15 are zero
    uint32_t qa[KS][4];
    auto load_q = [&](const auto& x) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int row = grp + 8 * rr;
            const bool row_in = row < gr;
            const __nv_bfloat16* qr =
                q + (static_cast<int64_t>(x.b) * H + x.h * rows + row_off + (row_in ? row : 0)) *
                        D;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qa[ks][rr] = row_in ? __ldg(reinterpret_cast<const uint32_t*>(qr + ks * 16 + 2 * tig)) : 0u;
                qa[ks][rr + 2] =
                    row_in ? __ldg(reinterpret_cast<const uint32_t*>(qr + ks * 16 + 8 + 2 * tig)) : 0u;
            }
        }
    };
    // piece kk from the producer; ntok < 0 ends the list
    struct Piece {
        int b, h, ntok, prow;
    };
    auto get_piece = [&](int kk, Piece& x) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.ud_full[kk & 1], (kk >> 1) & 1, err,
                                               FA_DEVERR_TIMEOUT, abort)))
            return false;
        const int* d = sm.ud[kk & 1];
        x.b = d[0];
        x.h = d[1];
        x.ntok = d[2];
        x.prow = d[3];
        mbar_arrive(&sm.ud_empty[kk & 1]);
        return true;
    };
    Piece us{0, 0, -1, 0};
    ok = get_piece(0, us);
    if (ok && us.ntok >= 0) load_q(us);
    for (; ok && us.ntok >= 0; ++k) {
        // rows grp (index 0) and grp + 8 (index 1, groups of 16 only)
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
        const int nchunks = (us.ntok + kGqTok - 1) / kGqTok;
        for (int c = 0; c < nchunks; ++c, ++g) {
            if ((g & 1) != crew) continue;
            const int slot = g % STAGES;
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[slot], (g / STAGES) & 1, err,
                                                   FA_DEVERR_TIMEOUT, abort));
            if (!ok) break;
            const uint32_t kb = smem_u32(sm.k[slot]), vb = smem_u32(sm.v[slot]);
            const int t0 = c * kGqTok + tbase;  // the warp's first token in the unit
            // ---- S = Q K^T: n-tile j holds tokens t0 + 8j .. +7; even and odd
            // k-steps accumulate apart (two chains of KS/2 products per n-tile)
            float s[NJ][4], s2[NJ][4];
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[j][e] = s2[j][e] = 0.f;
#pragma unroll
            for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    // matrices: column chunks 4kp .. 4kp+3 of token rows tbase + 8j ..
                    uint32_t b[4];
                    ldsm_x4(b, kb + gq_swz(tbase + 8 * j + lrow, 4 * kp + lmat));
                    mma_bf16_16816(s[j], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2],
                                   qa[2 * kp][3], b[0], b[1]);
                    mma_bf16_16816(s2[j], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2],
                                   qa[2 * kp + 1][3], b[2], b[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[j][e] += s2[j][e];
            // ---- online softmax of rows grp (and grp + 8) over this warp's WT tokens
            const bool partial = t0 + WT > us.ntok;
            uint32_t pa[KP][4];  // P as the A operand of k-step kk, as qa
#pragma unroll
            for (int rr = 0; rr < (kTwoRows ? 2 : 1); ++rr) {
                float sv[NJ][2];
#pragma unroll
                for (int j = 0; j < NJ; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) sv[j][e] = s[j][2 * rr + e] * scale_log2;
                if (partial) {
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            if (t0 + 8 * j + 2 * tig + e >= us.ntok) sv[j][e] = -INFINITY;
                }
                float mb = fmaxf(sv[0][0], sv[0][1]);
#pragma unroll
                for (int j = 1; j < NJ; ++j) mb = fmaxf(mb, fmaxf(sv[j][0], sv[j][1]));
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
                float pv[NJ][2];
#pragma unroll
                for (int j = 0; j < NJ; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) pv[j][e] = ex2_approx(sv[j][e] - mu);  // -inf -> 0
                float ps = 0.f;
#pragma unroll
                for (int j = 0; j < NJ; ++j) ps += pv[j][0] + pv[j][1];
                l[rr] += ps;
                m[rr] = mn;
                // k-step kk: tokens 2tig..+1 of n-tile 2kk (k columns 0-7)
                // and of n-tile 2kk+1 (8-15)
#pragma unroll
                for (int kk = 0; kk < KP; ++kk) {
                    pa[kk][rr] = pack_bf16x2(pv[2 * kk][0], pv[2 * kk][1]);
                    pa[kk][rr + 2] = pack_bf16x2(pv[2 * kk + 1][0], pv[2 * kk + 1][1]);
                }
            }
            if constexpr (!kTwoRows) {
#pragma unroll
                for (int kk = 0; kk < KP; ++kk) pa[kk][1] = pa[kk][3] = 0u;
            }
            // ---- O += P V: matrices (tokens 0-7 | 8-15 of k-step kk) x
            // (column chunk 2np | 2np+1).  V rows past the unit's tokens may
            // hold anything (0 * NaN): a partial slab zeroes their halves of
            // the B fragments
            auto pv_mma = [&](auto masked_c) {
                constexpr bool kMasked = decltype(masked_c)::value;
#pragma unroll
                for (int kk = 0; kk < KP; ++kk) {
                    uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
                    if constexpr (kMasked) {
                        const int tt = t0 + 16 * kk + 2 * tig;
                        mlo = (tt < us.ntok ? 0x0000ffffu : 0u) |
                              (tt + 1 < us.ntok ? 0xffff0000u : 0u);
                        mhi = (tt + 8 < us.ntok ? 0x0000ffffu : 0u) |
                              (tt + 9 < us.ntok ? 0xffff0000u : 0u);
                    }
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t b[4];
                        ldsm_x4_trans(b, vb + gq_swz(tbase + 16 * kk + 8 * (lmat & 1) + lrow,
                                                     2 * np + (lmat >> 1)));
                        if constexpr (kMasked) {
                            b[0] &= mlo;
                            b[1] &= mhi;
                            b[2] &= mlo;
                            b[3] &= mhi;
                        }
                        mma_bf16_16816(acc[2 * np], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3],
                                       b[0], b[1]);
                        mma_bf16_16816(acc[2 * np + 1], pa[kk][0], pa[kk][1], pa[kk][2],
                                       pa[kk][3], b[2], b[3]);
                    }
                }
            };
            if (partial) pv_mma(std::true_type{});
            else pv_mma(std::false_type{});
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[slot]);
        }
        if (!ok) break;
        // ---- merge the 8 warps' states of this unit in two rounds, once
        // every consumer has read the previous unit's merge out of the slots:
        // each warp of crew 1 hands its (m, l, O) to the crew-0 warp that
        // covers the same rows and tokens of the other chunks (same slot),
        // which folds it into its own and writes the pair's state back; then
        // all threads combine the slots of each set of rows
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
        auto put_state = [&]() {
#pragma unroll
            for (int rr = 0; rr < (kTwoRows ? 2 : 1); ++rr) {
                const int row = grp + 8 * rr;
                if (row < gr) {
                    if (tig == 0) {
                        sm.cm[row][mslot] = m[rr];
                        sm.cl[row][mslot] = l[rr];
                    }
#pragma unroll
                    for (int n = 0; n < NT; ++n)
                        *reinterpret_cast<float2*>(&sm.co[mslot][row][n * 8 + 2 * tig]) =
                            make_float2(acc[n][2 * rr], acc[n][2 * rr + 1]);
                }
            }
        };
        if (crew == 1) {
            put_state();
            mbar_arrive(&sm.c1);
        } else {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&sm.c1, k & 1, err, FA_DEVERR_TIMEOUT, abort));
            if (!ok) break;
#pragma unroll
            for (int rr = 0; rr < (kTwoRows ? 2 : 1); ++rr) {
                const int row = grp + 8 * rr;
                if (row < gr) {
                    const float mp = sm.cm[row][mslot], lp = sm.cl[row][mslot];
                    const float mx = fmaxf(m[rr], mp);
                    const float wa = (m[rr] == -INFINITY) ? 0.f : ex2_approx(m[rr] - mx);
                    const float wb = (mp == -INFINITY) ? 0.f : ex2_approx(mp - mx);
                    l[rr] = wa * l[rr] + wb * lp;
                    m[rr] = mx;
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const float2 c =
                            *reinterpret_cast<const float2*>(&sm.co[mslot][row][n * 8 + 2 * tig]);
                        acc[n][2 * rr] = wa * acc[n][2 * rr] + wb * c.x;
                        acc[n][2 * rr + 1] = wa * acc[n][2 * rr + 1] + wb * c.y;
                    }
                }
            }
            __syncwarp();  // every lane of the quad has read the partner's m and l
            put_state();
            mbar_arrive(&sm.cmb);
        }
        // the next piece, while the other warps merge (its query rows are
        // loaded after the combine: issued here they measured slower)
        Piece nx;
        ok = get_piece(k + 1, nx);
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.cmb, k & 1, err, FA_DEVERR_TIMEOUT, abort));
        if (!ok) break;
        // four columns of one query head per thread and pass: consecutive
        // threads read consecutive 16-byte words of a partial row; the passes
        // are independent, so they are unrolled (rows <= 2 GH)
        constexpr int D4 = D / 4;
        constexpr int kCombinePasses = (2 * GH * D4 + kGqWarps * 32 - 1) / (kGqWarps * 32);
#pragma unroll
        for (int it = 0; it < kCombinePasses; ++it) {
            const int idx = threadIdx.x + it * kGqWarps * 32;
            if (idx >= rows * D4) break;
            const int ha = idx / D4, x4 = idx - ha * D4;  // the unit's query head, column quad
            // the slots holding that head's states: its team's
            const int tt = kTwo ? ha / gr : 0;
            const int hi = ha - tt * gr;
            const int s0 = tt * kCrewWarps;
            float mw[kCrewWarps];
            float M = -INFINITY, L = 0.f;
#pragma unroll
            for (int w = 0; w < kCrewWarps; ++w) {
                mw[w] = sm.cm[hi][s0 + w];
                M = fmaxf(M, mw[w]);
            }
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kCrewWarps; ++w) {
                const float wgt = (mw[w] == -INFINITY) ? 0.f : ex2_approx(mw[w] - M);
                L += wgt * sm.cl[hi][s0 + w];
                const float4 c = *reinterpret_cast<const float4*>(&sm.co[s0 + w][hi][4 * x4]);
                o.x += wgt * c.x;
                o.y += wgt * c.y;
                o.z += wgt * c.z;
                o.w += wgt * c.w;
            }
            const float inv = 1.f / L;
            const int64_t pu = static_cast<int64_t>(us.prow) * rows + ha;
            *reinterpret_cast<float4*>(part_o + pu * D + 4 * x4) =
                make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
            if (x4 == 0) part_lse[pu] = M + __log2f(L);
        }
        if (nx.ntok >= 0) load_q(nx);
        us = nx;
        mbar_arrive(&sm.cfree);
    }
}

// One warp per (sequence, query head).  Sequence b's partials start at
// unit_off[b] * GH and are split-major with H per split.  Lane s holds the
// log-sum-exp of splits s and s + 32 (a sequence has at most 64), so the
// weights 2^(lse_s - M) come from one pass of loads and a shuffle each; the
// partial rows are then read as vectors, several splits in flight.
static_assert(kDecodeMaxSplits <= 64, "the merge holds two splits per lane");
template <int D>
__global__ void __launch_bounds__(128)
    fa_decode_merge_kernel(const int32_t* __restrict__ seq_lens, int B, int H, int GH,
                           int page_size, int max_splits, int min_pages,
                           const int32_t* __restrict__ unit_off,
                           const float* __restrict__ part_lse, const float* __restrict__ part_o,
                           __nv_bfloat16* __restrict__ o) {
    constexpr int PER = D / 32;  // columns per lane
    static_assert(PER == 2 || PER == 4, "64 or 128 columns");
    using Vec = typename std::conditional<PER == 4, float4, float2>::type;
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
    const float lse0 = lane < ns ? part_lse[base + lane * H + h] : -INFINITY;
    const float lse1 = lane + 32 < ns ? part_lse[base + (lane + 32) * H + h] : -INFINITY;
    float M = fmaxf(lse0, lse1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    // -inf - M -> weight 0 (an unused lane); M = -inf only when ns == 0
    const float w0 = ns > 0 ? ex2_approx(lse0 - M) : 0.f;
    const float w1 = ns > 0 ? ex2_approx(lse1 - M) : 0.f;
    float L = w0 + w1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int s = 0; s < ns; ++s) {
        const float w = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
        const int64_t unit = base + static_cast<int64_t>(s) * H + h;
        const Vec v = *reinterpret_cast<const Vec*>(part_o + unit * D + lane * PER);
        const float* vf = reinterpret_cast<const float*>(&v);
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, vf[i], acc[i]);
    }
    const float inv = ns > 0 ? 1.f / L : 0.f;
    __nv_bfloat16* dst = o + (static_cast<int64_t>(b) * H + h) * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2) {
        const uint32_t pk = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
        *reinterpret_cast<uint32_t*>(dst + i) = pk;
    }
}

// Grouped decode: one warp per (sequence, query head) merges the pieces of
// its slab (sequence b, unit head h / rows), rows slab_base[s] + j of rows
// query heads each, j over the CTAs the slab spans.  Lane j % 32 takes
// piece j's log-sum-exp in passes of 32; the weights reach the other lanes
// by shuffle.  An empty sequence gives zeros.
template <int D>
__global__ void __launch_bounds__(128)
    fa_decode_sk_merge_kernel(const int32_t* __restrict__ cnk_off, int B, int H, int Hk, int rows,
                              const int32_t* __restrict__ slab_base, int G,
                              const float* __restrict__ part_lse,
                              const float* __restrict__ part_o, __nv_bfloat16* __restrict__ o) {
    constexpr int PER = D / 32;  // columns per lane
    static_assert(PER == 2 || PER == 4, "64 or 128 columns");
    using Vec = typename std::conditional<PER == 4, float4, float2>::type;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= B * H) return;
    const int b = gw / H, hq = gw % H;
    const int h = hq / rows, ha = hq - h * rows;
    const int cb = __ldg(cnk_off + b), nc = __ldg(cnk_off + b + 1) - cb;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float L = 0.f;
    if (nc > 0) {
        const int64_t W = static_cast<int64_t>(Hk) * __ldg(cnk_off + B);
        G = sk_ctas(G, W);
        const int64_t start = static_cast<int64_t>(Hk) * cb + static_cast<int64_t>(h) * nc;
        const int np = sk_cta_of(start + nc - 1, W, G) - sk_cta_of(start, W, G) + 1;
        const int64_t base = __ldg(slab_base + b * Hk + h);
        float M = -INFINITY;
        for (int j = lane; j < np; j += 32) M = fmaxf(M, part_lse[(base + j) * rows + ha]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        for (int j0 = 0; j0 < np; j0 += 32) {
            const int n = min(32, np - j0);
            const float w = lane < n ? ex2_approx(part_lse[(base + j0 + lane) * rows + ha] - M) : 0.f;
            L += w;
#pragma unroll 4
            for (int jj = 0; jj < n; ++jj) {
                const float wj = __shfl_sync(0xffffffffu, w, jj);
                const int64_t r = (base + j0 + jj) * rows + ha;
                const Vec v = *reinterpret_cast<const Vec*>(part_o + r * D + lane * PER);
                const float* vf = reinterpret_cast<const float*>(&v);
#pragma unroll
                for (int i = 0; i < PER; ++i) acc[i] = fmaf(wj, vf[i], acc[i]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    }
    const float inv = nc > 0 ? 1.f / L : 0.f;
    __nv_bfloat16* dst = o + (static_cast<int64_t>(b) * H + hq) * D + lane * PER;
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

// Multi-head decode (one query head per K/V head): plan, split, merge.
template <int D>
int launch_decode_impl(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                       int num_pages,
                       int page_size, int max_splits, void* workspace, unsigned int* err,
                       int num_sms, cudaStream_t stream, uint64_t wait_ns = 0,
                       int withhold = 0) {
    const int rows = 1;  // query heads per unit
    const int Hk = H;    // units per split
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
    {
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
            err, wait_ns, withhold);
    }
    const int warps = B * H;
    fa_decode_merge_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(
        seq_lens, B, H, rows, page_size, max_splits, min_pages, unit_off, part_lse, part_o,
        static_cast<__nv_bfloat16*>(o));
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
// A group of G = H / Hk query heads per K/V head is cut into sub
// sub-groups of gr = G / sub heads, sub the fewest that leaves gr <= 16; an
// even number of sub-groups runs as pairs (teams == 2), one unit head per
// pair, both reading each chunk; sub counts the unit heads per K/V head.
struct GroupShape {
    int gr, sub, teams;
};
inline GroupShape group_shape(int H, int Hk) {
    const int G = H / Hk;
    int sub = (G + 15) / 16;
    while (G % sub != 0) ++sub;
    GroupShape gs;
    gs.gr = G / sub;
    gs.teams = (sub % 2 == 0) ? 2 : 1;
    gs.sub = sub / gs.teams;
    return gs;
}

// The grouped decode splits the stream evenly over the CTAs (balanced) when
// a sequence has at most kSkMaxUnitHeads unit heads; with more, the pool is
// large and split units taken in turn measured faster (8 and 16 K/V heads
// for 32 query heads: 3 % and 5 %), their CTAs reading the heads of the same
// pages at one time rather than each its own pages across the whole pool.
constexpr int kSkMaxUnitHeads = 2;

// Workspace of the grouped decode with unit heads Hk of rows query heads.
inline size_t gqa_workspace_bytes(int B, int Hk, int rows, int d, int max_splits, int num_sms) {
    return Hk <= kSkMaxUnitHeads ? sk_layout_of(B, Hk, rows, d, num_sms).total
                                 : layout_of(B, Hk * rows, d, max_splits).total;
}

// Grouped decode: plan, the grouped kernel on one CTA per SM (its shared
// memory admits no second), merge.
template <int D, int GH, int WT>
int launch_decode_gqa(const void* q, const CUtensorMap* tk, const CUtensorMap* tv,
                      const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                      int num_pages, int page_size, int max_splits, void* workspace,
                      size_t workspace_bytes, unsigned int* err, int num_sms, cudaStream_t stream,
                      int gr, int sub, int teams) {
    if (!tk || !tv) return FA_ERR_NULL;
    if (teams != WT / 16) return FA_ERR_UNSUPPORTED;
    const int rows = gr * teams;  // query heads per unit
    const int Hk = H / rows;      // unit heads per sequence
    auto split = fa_decode_gqa_kernel<D, GH, WT>;
    const size_t smem = sizeof(GqSmem<D, GH, WT>) + 1024;
    if (cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FA_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, split, kGqThreads, smem) !=
            cudaSuccess ||
        occ != 1)
        return FA_ERR_CUDA;
    const int G = num_sms;
    if (gqa_workspace_bytes(B, Hk, rows, D, max_splits, G) > workspace_bytes) return FA_ERR_SHAPE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const int warps = B * H;
    if (Hk <= kSkMaxUnitHeads) {
        const SkLayout L = sk_layout_of(B, Hk, rows, D, G);
        int32_t* page_off = reinterpret_cast<int32_t*>(ws + L.page_off);
        int32_t* cnk_off = reinterpret_cast<int32_t*>(ws + L.cnk_off);
        int32_t* slab_base = reinterpret_cast<int32_t*>(ws + L.slab_base);
        int32_t* first_slab = reinterpret_cast<int32_t*>(ws + L.first_slab);
        float* part_lse = reinterpret_cast<float*>(ws + L.lse_off);
        float* part_o = reinterpret_cast<float*>(ws + L.o_off);
        fa_decode_sk_plan_kernel<<<1, kPlanThreads, 0, stream>>>(
            seq_lens, B, Hk, G, page_off, cnk_off, slab_base, first_slab, err);
        split<<<G, kGqThreads, smem, stream>>>(
            *tk, *tv, static_cast<const __nv_bfloat16*>(q), page_table, seq_lens, B, H, Hk, gr,
            sub, num_pages, 1, page_off, cnk_off, slab_base, first_slab, nullptr, 0, 0, part_lse,
            part_o, scale_log2, err);
        fa_decode_sk_merge_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(
            cnk_off, B, H, Hk, rows, slab_base, G, part_lse, part_o,
            static_cast<__nv_bfloat16*>(o));
    } else {
        const int min_pages = Hk >= kDecodeManyUnits ? kDecodeChunkPages : kDecodeChunkPagesFew;
        const WorkspaceLayout L = layout_of(B, H, D, max_splits);
        int32_t* page_off = reinterpret_cast<int32_t*>(ws);
        int32_t* tok_off = page_off + (B + 1);
        int32_t* unit_off = tok_off + (B + 1);
        float* part_lse = reinterpret_cast<float*>(ws + L.lse_off);
        float* part_o = reinterpret_cast<float*>(ws + L.o_off);
        fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(
            seq_lens, B, Hk, page_size, max_splits, min_pages, page_off, tok_off, unit_off, err);
        split<<<G, kGqThreads, smem, stream>>>(
            *tk, *tv, static_cast<const __nv_bfloat16*>(q), page_table, seq_lens, B, H, Hk, gr,
            sub, num_pages, 0, page_off, nullptr, nullptr, nullptr, unit_off, max_splits,
            min_pages, part_lse, part_o, scale_log2, err);
        fa_decode_merge_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(
            seq_lens, B, H, rows, page_size, max_splits, min_pages, unit_off, part_lse, part_o,
            static_cast<__nv_bfloat16*>(o));
    }
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
                    int page_size, int max_splits, void* workspace, size_t workspace_bytes,
                    unsigned int* err, int num_sms, cudaStream_t stream) {
    if (H == Hk)
        return launch_decode_impl<D>(q, k_pages, v_pages, page_table, seq_lens, o, B, H,
                                     num_pages, page_size, max_splits, workspace, err, num_sms,
                                     stream);
    const GroupShape gs = group_shape(H, Hk);
#define FA_DECODE_GH(GH)                                                                        \
    if (gs.gr <= GH) {                                                                          \
        if (gs.teams == 2)                                                                      \
            return launch_decode_gqa<D, GH, 32>(q, tk, tv, page_table, seq_lens, o, B, H,       \
                                                num_pages, page_size, max_splits, workspace,    \
                                                workspace_bytes, err, num_sms, stream, gs.gr,   \
                                                gs.sub, 2);                                     \
        return launch_decode_gqa<D, GH, 16>(q, tk, tv, page_table, seq_lens, o, B, H,           \
                                            num_pages, page_size, max_splits, workspace,        \
                                            workspace_bytes, err, num_sms, stream, gs.gr,       \
                                            gs.sub, 1);                                         \
    }
    FA_DECODE_GH(2)
    FA_DECODE_GH(4)
    FA_DECODE_GH(8)
    FA_DECODE_GH(16)
#undef FA_DECODE_GH
    return FA_ERR_UNSUPPORTED;
}
}  // namespace

bool decode_group_supported(int H, int Hk) { return Hk >= 1 && H % Hk == 0; }

size_t decode_gqa_workspace_bytes(int B, int H, int Hk, int d, int max_splits, int num_sms) {
    const GroupShape gs = group_shape(H, Hk);
    const int rows = gs.gr * gs.teams;
    return gqa_workspace_bytes(B, H / rows, rows, d, max_splits, num_sms);
}

int launch_decode_stall(const void* q, const void* k_pages, const void* v_pages,
                        const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                        int d, int page_size, void* workspace, unsigned int* err, int num_sms,
                        cudaStream_t stream, uint64_t wait_ns, int withhold) {
    if (d == 128)
        return launch_decode_impl<128>(q, k_pages, v_pages, page_table,
                                       seq_lens, o, B, H, 0x7fffffff, page_size, kDecodeMaxSplits,
                                       workspace, err, num_sms, stream, wait_ns, withhold);
    if (d == 64)
        return launch_decode_impl<64>(q, k_pages, v_pages, page_table, seq_lens,
                                      o, B, H, 0x7fffffff, page_size, kDecodeMaxSplits, workspace,
                                      err, num_sms, stream, wait_ns, withhold);
    return FA_ERR_UNSUPPORTED;
}

int launch_decode(const void* q, const void* k_pages, const void* v_pages,
                  const CUtensorMap* tk, const CUtensorMap* tv, const int32_t* page_table,
                  const int32_t* seq_lens, void* o, int B, int H, int Hk, int num_pages, int d,
                  int page_size, int max_splits, void* workspace, size_t workspace_bytes,
                  unsigned int* err, int num_sms, cudaStream_t stream) {
    if (!decode_group_supported(H, Hk)) return FA_ERR_UNSUPPORTED;
    if (d == 128)
        return launch_decode_d<128>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, B, H,
                                    Hk, num_pages, page_size, max_splits, workspace,
                                    workspace_bytes, err, num_sms, stream);
    if (d == 64)
        return launch_decode_d<64>(q, k_pages, v_pages, tk, tv, page_table, seq_lens, o, B, H, Hk,
                                   num_pages, page_size, max_splits, workspace, workspace_bytes,
                                   err, num_sms, stream);
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
