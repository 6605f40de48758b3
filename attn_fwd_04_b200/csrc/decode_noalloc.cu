// decode_noalloc.cu -- fa_decode_paged_noalloc: paged decode that allocates
// nothing.
//
// Some callers cannot call cudaMalloc at all: a real-time serving loop whose
// memory was all reserved at start-up (an allocation could fail, or stall the
// loop while the allocator synchronises), or an embedding program with its own
// device allocator that forbids anyone else from allocating.  fa_decode_paged grows a library workspace on
// first use, which such callers cannot allow.  This entry point runs the same
// decode kernels with their scratch (split offsets and per-split partial
// outputs) in a fixed file-scope device array instead.
//
// The array is sized once, at compile time; every GPU that loads the library
// keeps it until the process exits.  All calls share it and it keeps the last
// call's contents; nothing in it has to start at zero (each call writes its
// offsets and partials before reading them).  Calls whose kernels overlap on
// the GPU -- on different streams without ordering, or from several threads --
// race on the array and give wrong results; order them.
#include <mutex>

#include "fa_internal.h"

namespace {

// 16 MiB: the partials of B*H*splits rows of d floats (+ offsets) must fit.
constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the name g_decode_scratch is only a host-side stand-in, never a device
// address, so the address is looked up once per device, with that device
// current, and cached.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
            return FA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FA_OK;
}

}  // namespace

extern "C" {

FA_API int fa_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* page_table, const int32_t* seq_lens, void* o,
                                   int B, int H, int d, int page_size, fa_stream_t stream) {
    if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !o) return FA_ERR_NULL;
    if (B < 1 || H < 1) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (page_size != 256) return FA_ERR_UNSUPPORTED;
    if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_pages) |
          reinterpret_cast<uintptr_t>(v_pages) | reinterpret_cast<uintptr_t>(o)) & 15u) != 0)
        return FA_ERR_ALIGN;
    // As many splits per sequence as the fixed scratch holds (at most the
    // allocating path's count); not even one split per (sequence, head) is
    // a size beyond this entry point's limit.
    int splits = 0;
    for (int s = fa::kDecodeMaxSplits; s >= 1; --s) {
        if (fa::decode_workspace_bytes(B, H, d, s) <= kScratchBytes) {
            splits = s;
            break;
        }
    }
    if (splits == 0) return FA_ERR_SHAPE;
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != FA_OK) return rc;
    unsigned int* err = nullptr;
    int num_sms = 0;
    if ((rc = fa::device_error_word(&err, &num_sms)) != FA_OK) return rc;
    // the signature carries no pool size: page indices are not bounded
    return fa::launch_decode(q, k_pages, v_pages, nullptr, nullptr, page_table, seq_lens, o, B, H,
                             H, 0x7fffffff, d, page_size, splits, scratch, kScratchBytes, err,
                             num_sms, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
