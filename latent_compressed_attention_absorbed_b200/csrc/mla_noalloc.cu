// mla_decode_no_alloc: the decode step for callers that cannot allocate
// device memory.
//
// Who needs it: a caller whose device memory belongs to someone else's
// allocator (an inference server or framework that owns the pool and does
// not let plug-in code call cudaMalloc), or a serving loop that must not
// allocate after start-up because cudaMalloc/cudaFree can synchronise the
// device and stall every stream.  Such a caller cannot hand mla_decode the
// workspace it needs.
//
// How: the workspace lives in a fixed array in this library's device image
// (kScratchBytes, 64 MiB).  Every GPU on which the library is loaded holds
// that array until the process exits.  The entry point passes the array to
// the ordinary decode path; it allocates nothing itself.
#include <cuda_runtime.h>

#include <mutex>

#include "mla_internal.h"

namespace {

// 64 MiB.  On a 148-SM B200 this holds the decode workspace of up to
// B * q_len = 88 query tokens: each token takes about 529 KiB (Q-hat, o_lat
// and one split-KV partial slot) on top of 74 fixed partial slots of
// 256.5 KiB.  Larger batches are rejected before anything is launched.
constexpr size_t kScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  The array's
// name in host code is only a host-side stand-in, so the address is looked
// up with cudaGetSymbolAddress once per device, with that device current.
int scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return mla::set_error(MLA_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices) return mla::set_error(MLA_ERR_ARG, "device index out of range");
    std::lock_guard<std::mutex> g(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr)
            return mla::set_error(MLA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MLA_OK;
}

}  // namespace

extern "C" int mla_decode_no_alloc(const mla_dims_t* dims, const void* q_nope, const void* q_rope,
                                   const void* W_UK, const void* W_UV, const mla_cache_t* cache,
                                   const int32_t* seqlens, int32_t B, int32_t q_len, void* out,
                                   mla_stream_t stream) {
    if (!dims) return mla::set_error(MLA_ERR_ARG, "dims is NULL");
    if (B < 0 || q_len < 1) return mla::set_error(MLA_ERR_ARG, "need B >= 0 and q_len >= 1");
    const size_t need = mla_workspace_bytes(dims, B, q_len);
    if (need > kScratchBytes)
        return mla::set_error(MLA_ERR_WORKSPACE,
                              "mla_decode_no_alloc: this batch needs %zu bytes of scratch but the static scratch "
                              "holds %zu; use mla_decode with a caller workspace or a smaller batch",
                              need, kScratchBytes);
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != MLA_OK) return rc;
    // Nothing in the scratch has to start at zero: the decode writes every
    // byte it later reads within the same call.
    return mla_decode(dims, q_nope, q_rope, W_UK, W_UV, cache, seqlens, B, q_len, out, scratch, kScratchBytes,
                      stream);
}
