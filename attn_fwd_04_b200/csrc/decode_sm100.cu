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
//   split  -- a persistent grid over the units; a unit attends its query to
//             the tokens of a few consecutive pages with the online softmax
//             (running max and normaliser, page "Flash Attention 是什么",
//             section 关键术语解析, item 4) and writes a normalised partial
//             output and its log-sum-exp;
//   merge  -- per (sequence, head), the log-sum-exp merge of the partials:
//             lse = M + log sum_s 2^(lse_s - M), o = sum_s 2^(lse_s - lse) o_s.
// All logs and exponents are base 2 inside the path (scale * log2 e folded
// into the query).
#include <cuda_bf16.h>

#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kSplitThreads = 128;
constexpr int kUnroll = 4;  // tokens in flight per half-warp and step

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

// One CTA (4 warps = 8 groups of LPT lanes) per work unit at a time.
// LPT = D / 8 lanes hold one token's row (8 bf16 = 16 bytes each).
template <int D>
__global__ void __launch_bounds__(kSplitThreads)
    fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ k_pages,
                           const __nv_bfloat16* __restrict__ v_pages,
                           const int32_t* __restrict__ page_table,
                           const int32_t* __restrict__ seq_lens, int B, int H, int page_size,
                           int max_splits, const int32_t* __restrict__ page_off,
                           const int32_t* __restrict__ unit_off, float* __restrict__ part_lse,
                           float* __restrict__ part_o, float scale_log2) {
    constexpr int LPT = D / 8;               // lanes per token
    constexpr int GPW = 32 / LPT;            // token groups per warp
    constexpr int G = (kSplitThreads / 32) * GPW;  // token groups per CTA
    __shared__ float sh_m[G], sh_l[G];
    __shared__ float sh_o[G][D];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane / LPT;              // group within the warp
    const int gl = lane % LPT;               // lane within the group
    const int grp = warp * GPW + sub;        // group within the CTA
    const unsigned gmask = (LPT == 32) ? 0xffffffffu : (((1u << LPT) - 1u) << (sub * LPT));

    const int total_units = __ldg(unit_off + B);
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
        const int b = find_owner(unit_off, B, u);
        const int r = u - __ldg(unit_off + b);
        const int s = r / H, h = r % H;
        int len = __ldg(seq_lens + b);
        if (len < 0) len = 0;
        const int np = (len + page_size - 1) / page_size;
        int ns, cp;
        split_shape(np, max_splits, ns, cp);
        const int tok0 = s * cp * page_size;
        const int tok1 = min(len, tok0 + cp * page_size);
        const int32_t* pt = page_table + __ldg(page_off + b);

        // this lane's 8 query values, pre-scaled into the log2 domain
        float qf[8];
        {
            const uint4 qu = *reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * H + h) * D + gl * 8);
            bf16x8_to_f32(qu, qf);
#pragma unroll
            for (int i = 0; i < 8; ++i) qf[i] *= scale_log2;
        }
        float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;

        for (int t0 = tok0 + grp; t0 < tok1; t0 += G * kUnroll) {
            uint4 kr[kUnroll], vr[kUnroll];
            bool valid[kUnroll];
#pragma unroll
            for (int x = 0; x < kUnroll; ++x) {
                const int t = t0 + x * G;
                valid[x] = t < tok1;
                if (valid[x]) {
                    const int page = __ldg(pt + t / page_size);
                    const int slot = t % page_size;
                    const int64_t row = (static_cast<int64_t>(page) * H + h) * page_size + slot;
                    kr[x] = ld_stream(k_pages + row * D + gl * 8);
                    vr[x] = ld_stream(v_pages + row * D + gl * 8);
                }
            }
            float sc[kUnroll];
#pragma unroll
            for (int x = 0; x < kUnroll; ++x) {
                float kf[8];
                bf16x8_to_f32(kr[x], kf);
                float dot = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], kf[i], dot);
#pragma unroll
                for (int o = LPT / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(gmask, dot, o);
                sc[x] = valid[x] ? dot : -INFINITY;
            }
            float mb = sc[0];
#pragma unroll
            for (int x = 1; x < kUnroll; ++x) mb = fmaxf(mb, sc[x]);
            const float m_new = fmaxf(m, mb);  // finite: sc[0] is always a valid token
            const float alpha = ex2_approx(m - m_new);
            l *= alpha;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
            for (int x = 0; x < kUnroll; ++x) {
                if (valid[x]) {
                    const float pw = ex2_approx(sc[x] - m_new);
                    l += pw;
                    float vf[8];
                    bf16x8_to_f32(vr[x], vf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = fmaf(pw, vf[i], acc[i]);
                }
            }
            m = m_new;
        }
        // combine the G groups of this CTA
        if (gl == 0) {
            sh_m[grp] = m;
            sh_l[grp] = l;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) sh_o[grp][gl * 8 + i] = acc[i];
        __syncthreads();
        if (threadIdx.x < D) {
            float M = -INFINITY;
#pragma unroll
            for (int g = 0; g < G; ++g) M = fmaxf(M, sh_m[g]);
            float L = 0.f, o = 0.f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float w = (sh_m[g] == -INFINITY) ? 0.f : ex2_approx(sh_m[g] - M);
                L += w * sh_l[g];
                o += w * sh_o[g][threadIdx.x];
            }
            part_o[static_cast<int64_t>(u) * D + threadIdx.x] = o / L;
            if (threadIdx.x == 0) part_lse[u] = M + __log2f(L);
        }
        __syncthreads();
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
    const int grid = num_sms * 16;
    fa_decode_split_kernel<D><<<grid, kSplitThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_pages),
        static_cast<const __nv_bfloat16*>(v_pages), page_table, seq_lens, B, H, page_size,
        max_splits, page_off, unit_off, part_lse, part_o, scale_log2);
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
