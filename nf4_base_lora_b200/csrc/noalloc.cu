// nf4_quantize_noalloc: the encoder with its scratch in a fixed device array
// compiled into the library, for callers that cannot allocate device memory.
//
// Scratch of the encoder: the fp32 first-level absmax of every 64-block and
// eight fp64 partial sums per 256 blocks.  Here it lives in g_quant_scratch, a
// file-scope __device__ array sized for kNoallocMaxBlocks blocks, which every
// GPU that loads the library keeps until the process exits.  Host code must
// not pass the symbol itself to a kernel (on the host it names a stand-in, not
// device memory): the device address is looked up with cudaGetSymbolAddress on
// every call, with the caller's device current.  The lookup is a host-side
// table read once the library's device code is loaded on that device, so
// nothing is cached across calls: after a cudaDeviceReset (which unloads the
// module, so the array may come back at another address) the next call finds
// the new address.
#include <cuda_runtime.h>

#include "nf4lora.h"
#include "kernels.h"

namespace nf4lora {

namespace {

constexpr int64_t kNoallocMaxBlocks = int64_t(1) << 22;                 // 268,435,456 weights
constexpr int64_t kNoallocMaxTiles = kNoallocMaxBlocks / 256;
constexpr int64_t kAbsmaxBytes = kNoallocMaxBlocks * 4;                  // 16 MiB
constexpr int64_t kScratchBytes = kAbsmaxBytes + kNoallocMaxTiles * 64 + 256;  // + 1 MiB of warp sums, segment sums

static __device__ __align__(256) unsigned char g_quant_scratch[kScratchBytes];

// Device address of g_quant_scratch on the current device.  The first call
// on a device may load the library's device code there (lazy module loading),
// which is why the first call should come before any stream capture.
cudaError_t scratch_address(void** out) { return cudaGetSymbolAddress(out, g_quant_scratch); }

}  // namespace

}  // namespace nf4lora

extern "C" int nf4_quantize_noalloc(const float* W, int64_t d_out, int64_t d_in, const nf4_tensor* out,
                                    void* stream) {
    using namespace nf4lora;
    // Same checks as nf4_quantize, minus the workspace, plus the size limit.
    if (W == nullptr || out == nullptr) return NF4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(W) & 15u) != 0) return NF4_ERR_MISALIGNED;
    const size_t packed = nf4_packed_bytes(d_out, d_in);
    if (packed == 0) return NF4_ERR_UNSUPPORTED_SHAPE;
    const bool fp32_scales = out->absmax != nullptr;  // no double quantisation: no scratch at all
    if (out->d_out != d_out || out->d_in != d_in || !out->codes ||
        (!fp32_scales && (!out->qscale || !out->scale2 || !out->scale_mean)))
        return NF4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out->codes) & 15u) ||
        (fp32_scales && (reinterpret_cast<uintptr_t>(out->absmax) & 15u)) ||
        (!fp32_scales &&
         ((reinterpret_cast<uintptr_t>(out->qscale) & 15u) || (reinterpret_cast<uintptr_t>(out->scale2) & 15u) ||
          (reinterpret_cast<uintptr_t>(out->scale_mean) & 3u))))
        return NF4_ERR_MISALIGNED;
    const int64_t n = d_out * d_in, n_blocks = n / 64;
    if (!fp32_scales && n_blocks > kNoallocMaxBlocks) return NF4_ERR_UNSUPPORTED_SHAPE;  // beyond the fixed scratch
    int dev = 0, major = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NF4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NF4_ERR_CUDA;
    if (major != 10) return NF4_ERR_DEVICE;
    if (fp32_scales) {
        const cudaError_t e = launch_nf4_quantize(W, n, out->codes, nullptr, nullptr, nullptr, out->absmax, nullptr,
                                                  sms, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
    }
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return NF4_ERR_CUDA;
    unsigned char* base = static_cast<unsigned char*>(scratch);
    // Every scratch word the kernels read is written earlier in the same call,
    // so nothing needs clearing between calls.
    const cudaError_t e = launch_nf4_quantize(W, n, out->codes, out->qscale, out->scale2, out->scale_mean,
                                              reinterpret_cast<float*>(base),
                                              reinterpret_cast<double*>(base + kAbsmaxBytes), sms,
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
