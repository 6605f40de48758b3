// api.cu -- the extern "C" boundary of libfa.so (declared in include/fa.h):
// argument checks, TMA tensor maps, the per-(GPU, stream) library workspaces and the
// device error word.  No kernel arithmetic lives here.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "fa_ptx.cuh"

namespace {

// Waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait the attention kernels use; the wait must give up and record
// FA_ERR_DEVICE_TIMEOUT instead of spinning forever.
__global__ void fa_selftest_wait_kernel(unsigned int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        fa::mbar_init(&bar, 1);
        fa::fence_mbar_init();
        fa::mbar_wait(&bar, 0, err, FA_DEVERR_TIMEOUT, nullptr);
    }
}

// First fault recorded by any kernel of this library on a device (see
// fa_get_device_error).  One copy per device: it lives in the module.
__device__ unsigned int g_device_error = 0;

constexpr int kMaxDevices = 64;

// One grow-only workspace per stream (decode partials, rotated K, backward
// scratch, page offsets): calls on different streams never share scratch.
struct StreamWorkspace {
    cudaStream_t stream = nullptr;
    void* ptr = nullptr;
    size_t bytes = 0;
};

struct DeviceState {
    bool init = false;
    int num_sms = 0;
    int cc_major = 0;
    unsigned int* err = nullptr;  // device address of g_device_error
    std::vector<StreamWorkspace> ws;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
// fixed-length forward with d = 128 and no RoPE on CTA pairs (fa_fwd_set_cta_pairs);
// off by default: on B200 at the 1000 W cap the pair kernel measured ~4% below
// the single-CTA kernel on the long-prefill workload
std::atomic<int> g_fwd_pairs{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int get_encode_fn() {
    if (g_encode) return FA_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return FA_OK;
}

// Current device's state, initialised on first use (caller holds g_mu).
int device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    DeviceState& s = g_dev[dev];
    if (!s.init) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FA_ERR_CUDA;
        s.num_sms = prop.multiProcessorCount;
        s.cc_major = prop.major;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return FA_ERR_CUDA;
        s.err = static_cast<unsigned int*>(p);
        s.init = true;
    }
    *out = &s;
    return FA_OK;
}

int lookup_device(DeviceState** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    int rc = device_state(out);
    if (rc != FA_OK) return rc;
    if ((*out)->cc_major != 10) return FA_ERR_UNSUPPORTED;  // sm_100 family only
    return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// bf16 tensor map over `dims` (innermost first) with byte strides for dims 1..2
// and a box of `box` elements; 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap* map, const void* base, const cuuint64_t dims[3],
             const cuuint64_t strides[2], const cuuint32_t box[3]) {
    if (get_encode_fn() != FA_OK) return FA_ERR_CUDA;
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// fp32 tensor map over `dims` with 128-byte swizzle (box inner extent 32
// floats = 128 bytes); used as the destination of bulk reduce-adds.
int make_map_f32(CUtensorMap* map, const void* base, const cuuint64_t dims[3],
                 const cuuint64_t strides[2], const cuuint32_t box[3]) {
    if (get_encode_fn() != FA_OK) return FA_ERR_CUDA;
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// The stream's grow-only workspace on this device, allocated (and, when it
// grows, freed) in the stream's own order.
int ensure_workspace(DeviceState* s, size_t bytes, cudaStream_t stream, void** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    StreamWorkspace* w = nullptr;
    for (StreamWorkspace& e : s->ws)
        if (e.stream == stream) w = &e;
    if (!w) {
        s->ws.push_back(StreamWorkspace{stream, nullptr, 0});
        w = &s->ws.back();
    }
    if (w->bytes < bytes) {
        if (w->ptr) {
            if (cudaFreeAsync(w->ptr, stream) != cudaSuccess) return FA_ERR_CUDA;
            w->ptr = nullptr;
            w->bytes = 0;
        }
        void* p = nullptr;
        if (cudaMallocAsync(&p, bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return FA_ERR_NOMEM;
        }
        w->ptr = p;
        w->bytes = bytes;
    }
    *out = w->ptr;
    return FA_OK;
}

// The packed sequences heaviest first into this stream's workspace (its
// first B ints), for the forward pass's seq_order; more than kSeqOrderMax
// sequences, or one, keep their order (null).  Paged prefill uses it (its
// sequences' cached lengths differ widely: 1.8 % faster on the paged-prefill
// workload); the variable-length forward pass measured no gain from it.
int order_sequences(DeviceState* s, const int32_t* cu_seqlens, const int32_t* ctx_lens, int B,
                    int causal, cudaStream_t stream, const int32_t** order) {
    *order = nullptr;
    if (B < 2 || B > fa::kSeqOrderMax) return FA_OK;
    void* ws = nullptr;
    int rc = ensure_workspace(s, sizeof(int32_t) * static_cast<size_t>(B), stream, &ws);
    if (rc != FA_OK) return rc;
    int32_t* o = static_cast<int32_t*>(ws);
    if ((rc = fa::launch_seq_order(cu_seqlens, ctx_lens, B, causal ? 1 : 0, o, stream)) != FA_OK)
        return rc;
    *order = o;
    return FA_OK;
}

}  // namespace

namespace fa {
int device_error_word(unsigned int** err, int* num_sms) {
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    *err = s->err;
    *num_sms = s->num_sms;
    return FA_OK;
}
}  // namespace fa

namespace {

// Fixed-length forward pass with H query heads and H_kv K/V heads; with
// rope_cos / rope_sin (tables of max_pos rows) Q and K are rotated first,
// once per position, into the stream's workspace.
int fwd_fixed(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
              int H_kv, int N, int d, int causal, float scale, fa_stream_t stream,
              const float* rope_cos = nullptr, const float* rope_sin = nullptr,
              int max_pos = 0, int withhold_copy = 0, uint64_t wait_ns = 0) {
    if ((rope_cos == nullptr) != (rope_sin == nullptr)) return FA_ERR_NULL;
    if (rope_cos && (max_pos < N || !aligned16(rope_cos) || !aligned16(rope_sin)))
        return max_pos < N ? FA_ERR_SHAPE : FA_ERR_ALIGN;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (B < 1 || H < 1 || H_kv < 1 || N < 1) return FA_ERR_SHAPE;
    if (H % H_kv != 0) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * H > 65535) return FA_ERR_SHAPE;
    if (N > 0x7fffffff - 128) return FA_ERR_SHAPE;
    if (!std::isfinite(scale)) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const void* k_use = k;
    const void* q_use = q;
    if (rope_cos) {
        // RoPE: Q and K rotated once per position by one row-kernel launch
        // into the stream's workspace; the forward kernel then reads them
        void* ws = nullptr;
        const size_t kbytes = static_cast<size_t>(B) * H_kv * N * d * 2;
        const size_t qbytes = static_cast<size_t>(B) * H * N * d * 2;
        if ((rc = ensure_workspace(s, kbytes + qbytes, st, &ws)) != FA_OK) return rc;
        void* kr = ws;
        void* qr = static_cast<uint8_t*>(ws) + kbytes;
        if ((rc = fa::launch_rope_rows(k, kr, static_cast<int64_t>(B) * H_kv, q, qr,
                                       static_cast<int64_t>(B) * H, rope_cos, rope_sin, N, d,
                                       s->num_sms, st)) != FA_OK)
            return rc;
        k_use = kr;
        q_use = qr;
    }
    // CTA pairs (2-SM products) load K in halves of 64 keys
    const bool pair = d == 128 && g_fwd_pairs.load() != 0;
    CUtensorMap tq, tk, tv;
    const cuuint64_t dims_q[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                  static_cast<cuuint64_t>(B) * H};
    const cuuint64_t dims_kv[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                   static_cast<cuuint64_t>(B) * H_kv};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(N) * d * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t box_k[3] = {64, pair ? 64u : 128u, 1};
    if ((rc = make_map(&tq, q_use, dims_q, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k_use, dims_kv, strides, box_k)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, dims_kv, strides, box)) != FA_OK) return rc;
    fa::FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.cu_seqlens = nullptr;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.N = N;
    p.total = 0;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.err = s->err;
    p.withhold_copy = withhold_copy;
    p.wait_ns = wait_ns;
    return fa::launch_fwd(p, tq, tk, tv, d, pair ? fa::kFixedPair : fa::kFixed, st);
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, int causal, float scale, fa_stream_t stream) {
    return fwd_fixed(q, k, v, o, lse, B, H, H, N, d, causal, scale, stream);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int H_kv, int N, int d, int causal, float scale, fa_stream_t stream) {
    return fwd_fixed(q, k, v, o, lse, B, H, H_kv, N, d, causal, scale, stream);
}

int fa_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse,
                const float* rope_cos, const float* rope_sin, int max_pos, int B, int H,
                int H_kv, int N, int d, int causal, float scale, fa_stream_t stream) {
    if (!rope_cos || !rope_sin) return FA_ERR_NULL;
    return fwd_fixed(q, k, v, o, lse, B, H, H_kv, N, d, causal, scale, stream, rope_cos,
                     rope_sin, max_pos);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
               int d, int causal, float scale, fa_stream_t stream) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
    if (B < 1 || H < 1 || N < 1 || H_kv < 1 || H % H_kv != 0) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * H > 65535) return FA_ERR_SHAPE;
    if (N > 0x7fffffff - 128) return FA_ERR_SHAPE;
    if (!std::isfinite(scale)) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    CUtensorMap tq, tk, tv, tdo;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(B) * H};
    const cuuint64_t dims_kv[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                   static_cast<cuuint64_t>(B) * H_kv};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(N) * d * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if ((rc = make_map(&tq, q, dims, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k, dims_kv, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, dims_kv, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tdo, dout, dims, strides, box)) != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, fa::bwd_workspace_bytes(B, H, N, d), st, &ws)) != FA_OK)
        return rc;
    // the fp32 dQ accumulator [B*H, N, d] in the workspace, reduced into by TMA
    CUtensorMap tdq;
    const cuuint64_t adims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                 static_cast<cuuint64_t>(B) * H};
    const cuuint64_t astrides[2] = {static_cast<cuuint64_t>(d) * 4,
                                    static_cast<cuuint64_t>(N) * d * 4};
    const cuuint32_t abox[3] = {32, 128, 1};
    if ((rc = make_map_f32(&tdq, static_cast<uint8_t*>(ws) + fa::bwd_dq_acc_offset(B, H, N), adims,
                           astrides, abox)) != FA_OK)
        return rc;
    return fa::launch_bwd(o, dout, lse, dq, dk, dv, tq, tk, tv, tdo, tdq, B, H, H_kv, N, d,
                          causal ? 1 : 0, scale, ws, s->err, s->num_sms, st);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
           int causal, float scale, fa_stream_t stream) {
    return fa_bwd_gqa(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, d, causal, scale, stream);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv, const int32_t* cu_seqlens,
                  int B, int H, int H_kv, int total, int max_seqlen, int d, int causal,
                  float scale, fa_stream_t stream) {
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !cu_seqlens)
        return FA_ERR_NULL;
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || total < 1 || max_seqlen < 1)
        return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (max_seqlen > 0x7fffffff - 128 || static_cast<int64_t>(total) * H > 0x7fffffff / 128)
        return FA_ERR_SHAPE;
    if (static_cast<int64_t>((max_seqlen + 127) / 128) * B * H_kv > 0x7fffffff)
        return FA_ERR_SHAPE;
    if (!std::isfinite(scale)) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    // packed [total, heads, d] as (d, heads, total), a box of 128 rows of one head
    CUtensorMap tq, tk, tv, tdo;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(total)};
    const cuuint64_t dims_kv[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv),
                                   static_cast<cuuint64_t>(total)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(H) * d * 2};
    const cuuint64_t strides_kv[2] = {static_cast<cuuint64_t>(d) * 2,
                                      static_cast<cuuint64_t>(H_kv) * d * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if ((rc = make_map(&tq, q, dims, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k, dims_kv, strides_kv, box)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, dims_kv, strides_kv, box)) != FA_OK) return rc;
    if ((rc = make_map(&tdo, dout, dims, strides, box)) != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, fa::bwd_workspace_bytes(1, H, total, d), st, &ws)) != FA_OK)
        return rc;
    // the fp32 dQ accumulator, head-major [H, total, d] in the workspace (a
    // tile's rows contiguous), reduced into by TMA
    CUtensorMap tdq;
    const cuuint64_t adims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(total),
                                 static_cast<cuuint64_t>(H)};
    const cuuint64_t astrides[2] = {static_cast<cuuint64_t>(d) * 4,
                                    static_cast<cuuint64_t>(total) * d * 4};
    const cuuint32_t abox[3] = {32, 128, 1};
    if ((rc = make_map_f32(&tdq, static_cast<uint8_t*>(ws) + fa::bwd_dq_acc_offset(1, H, total),
                           adims, astrides, abox)) != FA_OK)
        return rc;
    return fa::launch_bwd(o, dout, lse, dq, dk, dv, tq, tk, tv, tdo, tdq, B, H, H_kv, max_seqlen,
                          d, causal ? 1 : 0, scale, ws, s->err, s->num_sms, st, cu_seqlens,
                          total);
}

int fa_fwd_varlen_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int32_t* cu_seqlens, int B, int H, int H_kv, int total,
                      int max_seqlen, int d, int causal, float scale, fa_stream_t stream) {
    if (!q || !k || !v || !o || !lse || !cu_seqlens) return FA_ERR_NULL;
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || total < 1 || max_seqlen < 1)
        return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return FA_ERR_SHAPE;
    if (max_seqlen > 0x7fffffff - 128) return FA_ERR_SHAPE;
    if (!std::isfinite(scale)) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    CUtensorMap tq, tk, tv;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(total)};
    const cuuint64_t dims_kv[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv),
                                   static_cast<cuuint64_t>(total)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(H) * d * 2};
    const cuuint64_t strides_kv[2] = {static_cast<cuuint64_t>(d) * 2,
                                      static_cast<cuuint64_t>(H_kv) * d * 2};
    const cuuint32_t box[3] = {64, 1, 128};
    if ((rc = make_map(&tq, q, dims, strides, box)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k, dims_kv, strides_kv, box)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, dims_kv, strides_kv, box)) != FA_OK) return rc;
    fa::FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.cu_seqlens = cu_seqlens;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.N = max_seqlen;
    p.total = total;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.err = s->err;
    return fa::launch_fwd(p, tq, tk, tv, d, fa::kVarlen, reinterpret_cast<cudaStream_t>(stream));
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int32_t* cu_seqlens, int B, int H, int total, int max_seqlen, int d,
                  int causal, float scale, fa_stream_t stream) {
    return fa_fwd_varlen_gqa(q, k, v, o, lse, cu_seqlens, B, H, H, total, max_seqlen, d, causal,
                             scale, stream);
}

int fa_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                     const int32_t* page_table, const int32_t* seq_lens, const int32_t* cu_q,
                     void* o, float* lse, int B, int H, int H_kv, int total_q, int max_q,
                     int num_pages, int d, int page_size, int causal, float scale,
                     fa_stream_t stream) {
    if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !cu_q || !o || !lse)
        return FA_ERR_NULL;
    if (B < 1 || H < 1 || H_kv < 1 || total_q < 1 || max_q < 1 || num_pages < 1)
        return FA_ERR_SHAPE;
    if (H % H_kv != 0) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(num_pages) * H_kv > 0x7fffffff) return FA_ERR_SHAPE;
    if (max_q > 0x7fffffff - 256) return FA_ERR_SHAPE;
    if (!std::isfinite(scale)) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) ||
        !aligned16(lse))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    CUtensorMap tq, tk, tv;
    // queries: packed rows, as fa_fwd_varlen
    const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                                 static_cast<cuuint64_t>(total_q)};
    const cuuint64_t qstrides[2] = {static_cast<cuuint64_t>(d) * 2,
                                    static_cast<cuuint64_t>(H) * d * 2};
    const cuuint32_t qbox[3] = {64, 1, 128};
    // the page pool [P, H_kv, 256, d]: (d, slot, page * H_kv + head)
    const cuuint64_t kdims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(page_size),
                                 static_cast<cuuint64_t>(num_pages) * H_kv};
    const cuuint64_t kstrides[2] = {static_cast<cuuint64_t>(d) * 2,
                                    static_cast<cuuint64_t>(page_size) * d * 2};
    const cuuint32_t kbox[3] = {64, 128, 1};
    if ((rc = make_map(&tq, q, qdims, qstrides, qbox)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k_pages, kdims, kstrides, kbox)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v_pages, kdims, kstrides, kbox)) != FA_OK) return rc;
    fa::FwdParams p{};
    p.o = o;
    p.lse = lse;
    p.cu_seqlens = cu_q;
    p.B = B;
    p.H = H;
    p.H_kv = H_kv;
    p.page_table = page_table;
    p.ctx_lens = seq_lens;
    p.N = max_q;
    p.total = total_q;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.err = s->err;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = order_sequences(s, cu_q, seq_lens, B, causal, st, &p.seq_order)) != FA_OK)
        return rc;
    return fa::launch_fwd(p, tq, tk, tv, d, fa::kPaged, st);
}

}  // extern "C"

namespace {
// num_pages = 0x7fffffff: the pool size is unknown (fa_decode_paged's
// signature has none), page indices are not bounded.  max_pages > 0: the
// table is a block table [B, max_pages], packed into the workspace first.
int decode_impl(const void* q, const void* k_pages, const void* v_pages,
                const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                int H_kv, int num_pages, int d, int page_size, fa_stream_t stream,
                int max_pages = 0) {
    if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !o) return FA_ERR_NULL;
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || num_pages < 1) return FA_ERR_SHAPE;
    if (max_pages < 0 || static_cast<int64_t>(B) * max_pages > 0x7fffffff ||
        static_cast<int64_t>(max_pages) * page_size > 0x7fffffff)
        return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (!fa::decode_group_supported(H, H_kv)) return FA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * H * fa::kDecodeMaxSplits > 0x7fffffff) return FA_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o))
        return FA_ERR_ALIGN;
    const bool grouped = H != H_kv;
    if (grouped && static_cast<int64_t>(num_pages) * H_kv > 0x7fffffff) return FA_ERR_SHAPE;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    CUtensorMap tk, tv;
    if (grouped) {
        // the page pool [P, H_kv, 256, d] as (d, slot, page * H_kv + head)
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(page_size),
                                    static_cast<cuuint64_t>(num_pages) * H_kv};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                       static_cast<cuuint64_t>(page_size) * d * 2};
        const cuuint32_t box[3] = {64, 64, 1};
        if ((rc = make_map(&tk, k_pages, dims, strides, box)) != FA_OK) return rc;
        if ((rc = make_map(&tv, v_pages, dims, strides, box)) != FA_OK) return rc;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t need = grouped ? fa::decode_gqa_workspace_bytes(B, H, H_kv, d,
                                                                 fa::kDecodeMaxSplits, s->num_sms)
                                : fa::decode_workspace_bytes(B, H, d, fa::kDecodeMaxSplits);
    const size_t dec_bytes = (need + 255) & ~static_cast<size_t>(255);
    // block table: the packed table and the cut lengths follow the decode's own workspace
    const size_t pack_bytes =
        max_pages > 0 ? (static_cast<size_t>(B) * max_pages + B) * sizeof(int32_t) : 0;
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, dec_bytes + pack_bytes, st, &ws)) != FA_OK) return rc;
    const int32_t* table = page_table;
    const int32_t* lens = seq_lens;
    if (max_pages > 0) {
        int32_t* packed = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + dec_bytes);
        int32_t* cut = packed + static_cast<size_t>(B) * max_pages;
        if ((rc = fa::launch_decode_pack(page_table, max_pages, seq_lens, B, page_size, packed,
                                         cut, s->err, st)) != FA_OK)
            return rc;
        table = packed;
        lens = cut;
    }
    return fa::launch_decode(q, k_pages, v_pages, grouped ? &tk : nullptr,
                             grouped ? &tv : nullptr, table, lens, o, B, H, H_kv, num_pages, d,
                             page_size, fa::kDecodeMaxSplits, ws, dec_bytes, s->err, s->num_sms,
                             st);
}
}  // namespace

extern "C" {

int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                    const int32_t* page_table, const int32_t* seq_lens, void* o, int B, int H,
                    int d, int page_size, fa_stream_t stream) {
    return decode_impl(q, k_pages, v_pages, page_table, seq_lens, o, B, H, H, 0x7fffffff, d,
                       page_size, stream);
}

int fa_decode_paged_gqa(const void* q, const void* k_pages, const void* v_pages,
                        const int32_t* page_table, const int32_t* seq_lens, void* o, int B,
                        int H, int H_kv, int num_pages, int d, int page_size,
                        fa_stream_t stream) {
    return decode_impl(q, k_pages, v_pages, page_table, seq_lens, o, B, H, H_kv, num_pages, d,
                       page_size, stream);
}

int fa_decode_paged_strided(const void* q, const void* k_pages, const void* v_pages,
                            const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                            void* o, int B, int H, int H_kv, int num_pages, int d, int page_size,
                            fa_stream_t stream) {
    if (max_pages < 1) return block_table ? FA_ERR_SHAPE : FA_ERR_NULL;
    return decode_impl(q, k_pages, v_pages, block_table, seq_lens, o, B, H, H_kv, num_pages, d,
                       page_size, stream, max_pages);
}

int fa_gather_paged(const void* pages, const int32_t* page_table, const int32_t* seq_lens,
                    void* out, int B, int H, int d, int page_size, fa_stream_t stream) {
    if (!pages || !page_table || !seq_lens || !out) return FA_ERR_NULL;
    if (B < 1 || H < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (!aligned16(pages) || !aligned16(out)) return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, fa::decode_workspace_bytes(B, H, d, 1), st, &ws)) != FA_OK)
        return rc;
    return fa::launch_gather(pages, page_table, seq_lens, out, B, H, d, page_size, ws, s->err,
                             s->num_sms, st);
}

int fa_append_paged(const void* k_new, const void* v_new, const int32_t* cu_new, void* k_pages,
                    void* v_pages, const int32_t* page_table, const int32_t* seq_lens, int B,
                    int H_kv, int total_new, int num_pages, int d, int page_size,
                    fa_stream_t stream) {
    if (!k_new || !v_new || !cu_new || !k_pages || !v_pages || !page_table || !seq_lens)
        return FA_ERR_NULL;
    if (B < 1 || H_kv < 1 || total_new < 0 || num_pages < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pages) || !aligned16(v_pages))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    if (total_new == 0) return FA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, fa::decode_workspace_bytes(B, H_kv, d, 1), st, &ws)) != FA_OK)
        return rc;
    return fa::launch_append(k_new, v_new, cu_new, k_pages, v_pages, page_table, seq_lens, B,
                             H_kv, total_new, d, page_size, num_pages, ws, s->err, s->num_sms,
                             st);
}

int fa_get_device_error(int* code, fa_stream_t stream) {
    if (!code) return FA_ERR_NULL;
    DeviceState* s = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int rc = device_state(&s);
        if (rc != FA_OK) return rc;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    const unsigned int zero = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpy(&v, s->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpy(s->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return FA_ERR_CUDA;
    *code = -static_cast<int>(v);
    return FA_OK;
}

int fa_selftest_bounded_wait(fa_stream_t stream) {
    DeviceState* s = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int rc = device_state(&s);
        if (rc != FA_OK) return rc;
    }
    fa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(s->err);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_selftest_fwd_stall(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, int withheld, int wait_us,
                          fa_stream_t stream) {
    if (withheld < 0 || wait_us < 1 || wait_us > 2000000) return FA_ERR_SHAPE;
    // the single-CTA kernel (the CTA-pair variant is not selected here)
    const int prev = g_fwd_pairs.exchange(0);
    const int rc = fwd_fixed(q, k, v, o, lse, B, H, H, N, d, 1, 1.f / std::sqrt(float(d)),
                             stream, nullptr, nullptr, 0, withheld + 1,
                             static_cast<uint64_t>(wait_us) * 1000u);
    g_fwd_pairs.store(prev);
    return rc;
}

int fa_selftest_decode_stall(const void* q, const void* k_pages, const void* v_pages,
                             const int32_t* page_table, const int32_t* seq_lens, void* o, int B,
                             int H, int d, int page_size, int withheld, int wait_us,
                             fa_stream_t stream) {
    if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !o) return FA_ERR_NULL;
    if (withheld < 0 || wait_us < 1 || wait_us > 2000000) return FA_ERR_SHAPE;
    if (B < 1 || H < 1 || static_cast<int64_t>(B) * H * fa::kDecodeMaxSplits > 0x7fffffff)
        return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o))
        return FA_ERR_ALIGN;
    DeviceState* s = nullptr;
    int rc = lookup_device(&s);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    if ((rc = ensure_workspace(s, fa::decode_workspace_bytes(B, H, d, fa::kDecodeMaxSplits), st,
                               &ws)) != FA_OK)
        return rc;
    return fa::launch_decode_stall(q, k_pages, v_pages, page_table, seq_lens, o, B, H, d,
                                   page_size, ws, s->err, s->num_sms, st,
                                   static_cast<uint64_t>(wait_us) * 1000u, withheld + 1);
}

int fa_release_workspace(void) {
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_OK;
    DeviceState& s = g_dev[dev];
    if (!s.ws.empty()) {
        if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
        for (StreamWorkspace& w : s.ws)
            if (w.ptr && cudaFree(w.ptr) != cudaSuccess) return FA_ERR_CUDA;
        s.ws.clear();
    }
    return FA_OK;
}

const char* fa_status_str(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
        case FA_ERR_SHAPE: return "FA_ERR_SHAPE: a size is out of range";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim, page size or device";
        case FA_ERR_ALIGN: return "FA_ERR_ALIGN: a tensor pointer is not 16-byte aligned";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call or launch failed";
        case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
        case FA_ERR_NOMEM: return "FA_ERR_NOMEM: workspace allocation failed";
        case FA_ERR_DEVICE_BAD_INPUT: return "FA_ERR_DEVICE_BAD_INPUT: invalid device-side input (negative length)";
        default: return "unknown fa status";
    }
}

int fa_version(void) { return 100; }

int fa_fwd_set_cta_pairs(int enable) { return g_fwd_pairs.exchange(enable ? 1 : 0); }

}  // extern "C"
