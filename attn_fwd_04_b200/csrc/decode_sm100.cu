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

// Splits of a sequence with np pages: at least kDecodeChunkPages pages each,
// at most max_splits of them, none empty.
__device__ __forceinline__ void split_shape(int np, int max_splits, int& ns, int& cp) {
    if (np <= 0) {
        ns = 0;
        cp = 1;
        return;
    }
    int want = (np + kDecodeChunkPages - 1) / kDecodeChunkPages;
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
                          int max_splits, int32_t* page_off, int32_t* tok_off, int32_t* unit_off,
                          unsigned int* err) {
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
        split_shape(np, max_splits, ns, cp);
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

__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

constexpr int kDecTok = 64;           // tokens per ring stage (a quarter of a page)
constexpr int kDecStages = 6;         // ring depth
constexpr int kDecConsumerWarps = 8;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;  // + one producer warp

template <int D>
struct DecSmem {
    static constexpr int LPT = D / 8;                              // lanes per token
    static constexpr int G = kDecConsumerWarps * 32 / LPT;         // token groups
    alignas(128) uint8_t k[kDecStages][kDecTok * D * 2];
    alignas(128) uint8_t v[kDecStages][kDecTok * D * 2];
    float cm[2][G], cl[2][G];          // per-group partial state, by unit parity
    float co[2][G][D];
    uint64_t full[kDecStages], empty[kDecStages], cmb[2];
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
    int b, s, h, tok0, ntok, cp, pt_base;
};

__device__ __forceinline__ UnitShape unit_shape(int u, UnitCursor& cur,
                                                const int32_t* __restrict__ unit_off,
                                                const int32_t* __restrict__ page_off,
                                                const int32_t* __restrict__ seq_lens, int B,
                                                int H, int page_size, int max_splits) {
    cur.seek(unit_off, B, u);
    UnitShape us;
    us.b = cur.b;
    const int r = u - __ldg(unit_off + us.b);
    us.s = r / H;
    us.h = r % H;
    int len = __ldg(seq_lens + us.b);
    if (len < 0) len = 0;
    const int np = (len + page_size - 1) / page_size;
    int ns;
    split_shape(np, max_splits, ns, us.cp);
    us.tok0 = us.s * us.cp * page_size;
    us.ntok = min(len, us.tok0 + us.cp * page_size) - us.tok0;
    us.pt_base = __ldg(page_off + us.b) + us.s * us.cp;
    return us;
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ k_pages,
                           const __nv_bfloat16* __restrict__ v_pages,
                           const int32_t* __restrict__ page_table,
                           const int32_t* __restrict__ seq_lens, int B, int H, int page_size,
                           int max_splits, const int32_t* __restrict__ page_off,
                           const int32_t* __restrict__ unit_off, float* __restrict__ part_lse,
                           float* __restrict__ part_o, float scale_log2, unsigned int* err) {
    using Sm = DecSmem<D>;
    constexpr int LPT = Sm::LPT, G = Sm::G;
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
                                            page_size, max_splits);
            const int nchunks = (us.ntok + kDecTok - 1) / kDecTok;
            constexpr int per_page = 256 / kDecTok;  // page_size is 256
            int page = 0;
            for (int c = 0; c < nchunks; ++c, ++g) {
                if (c % per_page == 0) page = __ldg(page_table + us.pt_base + c / per_page);
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
                                            page_size, max_splits);
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

// One warp per (sequence, head).
template <int D>
__global__ void __launch_bounds__(128)
    fa_decode_merge_kernel(const int32_t* __restrict__ seq_lens, int B, int H, int page_size,
                           int max_splits, const int32_t* __restrict__ unit_off,
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
    split_shape(np, max_splits, ns, cp);
    const int base = __ldg(unit_off + b);
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

template <int D>
int launch_decode_impl(const void* q, const void* k_pages, const void* v_pages,
                       const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                       int page_size, int max_splits, void* workspace, unsigned int* err,
                       int num_sms, cudaStream_t stream) {
    const WorkspaceLayout L = layout_of(B, H, D, max_splits);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* page_off = reinterpret_cast<int32_t*>(ws);
    int32_t* tok_off = page_off + (B + 1);
    int32_t* unit_off = tok_off + (B + 1);
    float* part_lse = reinterpret_cast<float*>(ws + L.lse_off);
    float* part_o = reinterpret_cast<float*>(ws + L.o_off);
    fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, B, H, page_size, max_splits,
                                                          page_off, tok_off, unit_off, err);
    const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
    const size_t smem = sizeof(DecSmem<D>) + 128;
    if (cudaFuncSetAttribute(fa_decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FA_ERR_CUDA;
    // a persistent grid of the CTAs that are resident at once
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fa_decode_split_kernel<D>,
                                                      kDecThreads, smem) != cudaSuccess ||
        occ < 1)
        return FA_ERR_CUDA;
    fa_decode_split_kernel<D><<<num_sms * occ, kDecThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_pages),
        static_cast<const __nv_bfloat16*>(v_pages), page_table, seq_lens, B, H, page_size,
        max_splits, page_off, unit_off, part_lse, part_o, scale_log2, err);
    const int warps = B * H;
    fa_decode_merge_kernel<D><<<(warps + 3) / 4, 128, 0, stream>>>(
        seq_lens, B, H, page_size, max_splits, unit_off, part_lse, part_o,
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
    fa_decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(seq_lens, B, H, page_size, 1, page_off,
                                                          tok_off, unit_off, err);
    fa_gather_kernel<D><<<num_sms * 8, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(pages), page_table, seq_lens, B, H, page_size,
        page_off, tok_off, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

size_t decode_workspace_bytes(int B, int H, int d, int max_splits) {
    return layout_of(B, H, d, max_splits).total;
}

int launch_decode(const void* q, const void* k_pages, const void* v_pages,
                  const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                  int d, int page_size, int max_splits, void* workspace, unsigned int* err,
                  int num_sms, cudaStream_t stream) {
    if (d == 128)
        return launch_decode_impl<128>(q, k_pages, v_pages, page_table, seq_lens, o, B, H,
                                       page_size, max_splits, workspace, err, num_sms, stream);
    if (d == 64)
        return launch_decode_impl<64>(q, k_pages, v_pages, page_table, seq_lens, o, B, H,
                                      page_size, max_splits, workspace, err, num_sms, stream);
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
