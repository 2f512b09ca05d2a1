// C ABI of libnf4lora: argument checks, workspace sizing and dispatch.
// Declarations and the meaning of every argument: include/nf4lora.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "nf4lora.h"
#include "common.cuh"
#include "kernels.h"
#include "layer.h"

namespace nf4lora {
__device__ int g_device_status = 0;
__device__ unsigned int g_debug_site = 0;
}

using namespace nf4lora;

namespace {

thread_local std::string t_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

int ok() {
    t_last_error.clear();
    return NF4_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t align256(int64_t b) { return (b + 255) & ~int64_t(255); }

bool valid_weight_shape(int64_t d_out, int64_t d_in) {
    return d_out >= 1 && d_in >= 64 && d_in % 64 == 0 && d_out < (int64_t(1) << 31) &&
           d_in < (int64_t(1) << 31);
}

// Current device must be a B200-class part (compute capability 10.x).
int check_device(int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(NF4_ERR_CUDA, "cudaGetDevice failed");
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return fail(NF4_ERR_CUDA, "cudaDeviceGetAttribute failed");
    if (major != 10) return fail(NF4_ERR_DEVICE, "device %d has compute capability %d.x; sm_100 required", dev, major);
    *num_sms = sms;
    return NF4_OK;
}

int check_tensor(const nf4_tensor* w) {
    if (w == nullptr) return fail(NF4_ERR_INVALID_ARG, "nf4_tensor is NULL");
    if (!valid_weight_shape(w->d_out, w->d_in))
        return fail(NF4_ERR_UNSUPPORTED_SHAPE, "weight [%lld, %lld]: need d_out >= 1, d_in >= 64, d_in %% 64 == 0",
                    (long long)w->d_out, (long long)w->d_in);
    if (w->absmax != nullptr) {
        // fp32 block scales, no double quantisation
        if (!w->codes) return fail(NF4_ERR_INVALID_ARG, "nf4_tensor has NULL codes");
        if (!aligned16(w->codes) || !aligned16(w->absmax))
            return fail(NF4_ERR_MISALIGNED, "nf4_tensor member not aligned (codes/absmax: 16 B)");
        return NF4_OK;
    }
    if (!w->codes || !w->qscale || !w->scale2 || !w->scale_mean)
        return fail(NF4_ERR_INVALID_ARG, "nf4_tensor has a NULL member");
    if (!aligned16(w->codes) || !aligned16(w->qscale) || !aligned16(w->scale2) ||
        (reinterpret_cast<uintptr_t>(w->scale_mean) & 3u))
        return fail(NF4_ERR_MISALIGNED, "nf4_tensor member not aligned (codes/qscale/scale2: 16 B, scale_mean: 4 B)");
    return NF4_OK;
}

int64_t quant_ws_bytes(int64_t d_out, int64_t d_in) {
    const int64_t nb = d_out * d_in / 64;
    const int64_t tiles = (nb + 255) / 256;
    const int64_t segs = (tiles + 2047) / 2048;
    // absmax; 8 fp64 warp sums per tile, the fp64 segment sums and a ticket
    return align256(nb * 4) + align256(tiles * 8 * 8 + segs * 8 + 8);
}

int check_layer_common(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling,
                       int64_t M) {
    int rc = check_tensor(w);
    if (rc) return rc;
    if (w->d_out % 8 != 0) return fail(NF4_ERR_UNSUPPORTED_SHAPE, "d_out = %lld must be a multiple of 8", (long long)w->d_out);
    if (r < 1 || r > 256) return fail(NF4_ERR_INVALID_ARG, "r = %d outside [1, 256]", r);
    if (!std::isfinite(scaling)) return fail(NF4_ERR_INVALID_ARG, "scaling is not finite");
    if (M < 0 || M >= (int64_t(1) << 31)) return fail(NF4_ERR_INVALID_ARG, "M = %lld outside [0, 2^31)", (long long)M);
    if (!A || !B) return fail(NF4_ERR_INVALID_ARG, "A or B is NULL");
    if (!aligned16(A) || !aligned16(B)) return fail(NF4_ERR_MISALIGNED, "A or B not 16-byte aligned");
    return NF4_OK;
}

int check_ws(void* ws, size_t ws_bytes, int64_t need) {
    if (need <= 0) return NF4_OK;
    if (ws == nullptr) return fail(NF4_ERR_WORKSPACE, "workspace is NULL (%lld bytes needed)", (long long)need);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(NF4_ERR_MISALIGNED, "workspace not 256-byte aligned");
    if (static_cast<int64_t>(ws_bytes) < need)
        return fail(NF4_ERR_WORKSPACE, "workspace of %zu bytes < %lld needed", ws_bytes, (long long)need);
    return NF4_OK;
}

}  // namespace

extern "C" {

size_t nf4_packed_bytes(int64_t d_out, int64_t d_in) {
    if (!valid_weight_shape(d_out, d_in)) return 0;
    const int64_t n = d_out * d_in, nb = n / 64, ng = (nb + 255) / 256;
    return static_cast<size_t>(align256(n / 2) + align256(nb) + align256(ng * 4) + 256);
}

int nf4_tensor_from_buffer(nf4_tensor* t, void* base, size_t bytes, int64_t d_out, int64_t d_in) {
    if (t == nullptr || base == nullptr) return fail(NF4_ERR_INVALID_ARG, "NULL tensor or buffer");
    if (!valid_weight_shape(d_out, d_in))
        return fail(NF4_ERR_UNSUPPORTED_SHAPE, "weight [%lld, %lld]: need d_in %% 64 == 0", (long long)d_out, (long long)d_in);
    if (reinterpret_cast<uintptr_t>(base) & 255u) return fail(NF4_ERR_MISALIGNED, "buffer not 256-byte aligned");
    if (bytes < nf4_packed_bytes(d_out, d_in)) return fail(NF4_ERR_INVALID_ARG, "buffer too small");
    const int64_t n = d_out * d_in, nb = n / 64, ng = (nb + 255) / 256;
    uint8_t* p = static_cast<uint8_t*>(base);
    t->d_out = d_out;
    t->d_in = d_in;
    t->codes = p;
    p += align256(n / 2);
    t->qscale = reinterpret_cast<int8_t*>(p);
    p += align256(nb);
    t->scale2 = reinterpret_cast<float*>(p);
    p += align256(ng * 4);
    t->scale_mean = reinterpret_cast<float*>(p);
    t->absmax = nullptr;
    return ok();
}

size_t nf4_packed_bytes_nodq(int64_t d_out, int64_t d_in) {
    if (!valid_weight_shape(d_out, d_in)) return 0;
    const int64_t n = d_out * d_in, nb = n / 64;
    return static_cast<size_t>(align256(n / 2) + align256(nb * 4));
}

int nf4_tensor_from_buffer_nodq(nf4_tensor* t, void* base, size_t bytes, int64_t d_out, int64_t d_in) {
    if (t == nullptr || base == nullptr) return fail(NF4_ERR_INVALID_ARG, "NULL tensor or buffer");
    if (!valid_weight_shape(d_out, d_in))
        return fail(NF4_ERR_UNSUPPORTED_SHAPE, "weight [%lld, %lld]: need d_in %% 64 == 0", (long long)d_out, (long long)d_in);
    if (reinterpret_cast<uintptr_t>(base) & 255u) return fail(NF4_ERR_MISALIGNED, "buffer not 256-byte aligned");
    if (bytes < nf4_packed_bytes_nodq(d_out, d_in)) return fail(NF4_ERR_INVALID_ARG, "buffer too small");
    const int64_t n = d_out * d_in;
    uint8_t* p = static_cast<uint8_t*>(base);
    t->d_out = d_out;
    t->d_in = d_in;
    t->codes = p;
    t->qscale = nullptr;
    t->scale2 = nullptr;
    t->scale_mean = nullptr;
    t->absmax = reinterpret_cast<float*>(p + align256(n / 2));
    return ok();
}

size_t nf4_quantize_workspace_bytes(int64_t d_out, int64_t d_in) {
    if (!valid_weight_shape(d_out, d_in)) return 0;
    return static_cast<size_t>(quant_ws_bytes(d_out, d_in));
}

size_t qlora_fwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r) {
    if (!valid_weight_shape(d_out, d_in) || M < 1 || r < 1 || r > 256) return 0;
    return static_cast<size_t>(fwd_workspace_bytes(M, d_out, d_in, r, kPlanSMs));
}

size_t qlora_bwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r) {
    if (!valid_weight_shape(d_out, d_in) || M < 1 || r < 1 || r > 256) return 0;
    return static_cast<size_t>(bwd_workspace_bytes(M, d_out, d_in, r, kPlanSMs));
}

int nf4_quantize(const float* W, int64_t d_out, int64_t d_in, const nf4_tensor* out, void* ws, size_t ws_bytes,
                 void* stream) {
    if (W == nullptr) return fail(NF4_ERR_INVALID_ARG, "W is NULL");
    if (!aligned16(W)) return fail(NF4_ERR_MISALIGNED, "W not 16-byte aligned");
    int rc = check_tensor(out);
    if (rc) return rc;
    if (out->d_out != d_out || out->d_in != d_in)
        return fail(NF4_ERR_INVALID_ARG, "out describes [%lld, %lld], W is [%lld, %lld]", (long long)out->d_out,
                    (long long)out->d_in, (long long)d_out, (long long)d_in);
    const int64_t n = d_out * d_in, nb = n / 64;
    if (out->absmax != nullptr) {
        // fp32 block scales: the encoder writes them directly, no workspace
        int sms = 0;
        rc = check_device(&sms);
        if (rc) return rc;
        cudaError_t e = launch_nf4_quantize(W, n, out->codes, nullptr, nullptr, nullptr, out->absmax, nullptr, sms,
                                            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_quantize launch: %s", cudaGetErrorString(e));
        return ok();
    }
    rc = check_ws(ws, ws_bytes, quant_ws_bytes(d_out, d_in));
    if (rc) return rc;
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    float* absmax = reinterpret_cast<float*>(w8);
    double* tile_sums = reinterpret_cast<double*>(w8 + align256(nb * 4));
    cudaError_t e = launch_nf4_quantize(W, n, out->codes, out->qscale, out->scale2, out->scale_mean, absmax, tile_sums,
                                        sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_quantize launch: %s", cudaGetErrorString(e));
    return ok();
}

int nf4_dequantize(const nf4_tensor* w, uint16_t* W_hat, void* stream) {
    int rc = check_tensor(w);
    if (rc) return rc;
    if (W_hat == nullptr) return fail(NF4_ERR_INVALID_ARG, "W_hat is NULL");
    if (!aligned16(W_hat)) return fail(NF4_ERR_MISALIGNED, "W_hat not 16-byte aligned");
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    cudaError_t e = launch_nf4_dequantize(w->codes, w->qscale, w->scale2, w->scale_mean, w->absmax,
                                          w->d_out * w->d_in, W_hat, sms, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_dequantize launch: %s", cudaGetErrorString(e));
    return ok();
}

int qlora_linear_fwd(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling,
                     const uint16_t* X, int64_t M, uint16_t* Y, float* T_saved, void* ws, size_t ws_bytes,
                     void* stream) {
    int rc = check_layer_common(w, A, B, r, scaling, M);
    if (rc) return rc;
    if (M == 0) return ok();  // an empty batch
    if (!X || !Y) return fail(NF4_ERR_INVALID_ARG, "X or Y is NULL");
    if (!aligned16(X) || !aligned16(Y) || (T_saved && !aligned16(T_saved)))
        return fail(NF4_ERR_MISALIGNED, "X, Y or T_saved not 16-byte aligned");
    rc = check_ws(ws, ws_bytes, fwd_workspace_bytes(M, w->d_out, w->d_in, r, kPlanSMs));
    if (rc) return rc;
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    LayerCtx c{w->codes, w->qscale, w->scale2, w->scale_mean, w->absmax, w->d_out, w->d_in, kPlanSMs,
               static_cast<cudaStream_t>(stream)};
    rc = layer_fwd(c, A, B, r, scaling, X, M, Y, T_saved, static_cast<uint8_t*>(ws));
    if (rc == -1) return fail(NF4_ERR_CUDA, "qlora_linear_fwd: tensor map encoding failed");
    if (rc) return fail(NF4_ERR_CUDA, "qlora_linear_fwd launch: %s", cudaGetErrorString(layer_last_cuda_error()));
    return ok();
}

int qlora_linear_bwd(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling,
                     const uint16_t* X, const float* T_saved, const uint16_t* dY, int64_t M, uint16_t* dX,
                     uint16_t* dA, uint16_t* dB, int accumulate_grads, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_layer_common(w, A, B, r, scaling, M);
    if (rc) return rc;
    if (accumulate_grads != 0 && accumulate_grads != 1) return fail(NF4_ERR_INVALID_ARG, "accumulate_grads must be 0 or 1");
    if (M == 0) {
        // an empty batch: zero gradients for the adapters, nothing else
        if (accumulate_grads || (!dA && !dB)) return ok();
        if ((dA && !aligned16(dA)) || (dB && !aligned16(dB)))
            return fail(NF4_ERR_MISALIGNED, "dA or dB not 16-byte aligned");
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        if (dA && cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * w->d_in * 2, st) != cudaSuccess)
            return fail(NF4_ERR_CUDA, "qlora_linear_bwd: clearing dA failed");
        if (dB && cudaMemsetAsync(dB, 0, static_cast<size_t>(w->d_out) * r * 2, st) != cudaSuccess)
            return fail(NF4_ERR_CUDA, "qlora_linear_bwd: clearing dB failed");
        return ok();
    }
    if (!dY) return fail(NF4_ERR_INVALID_ARG, "dY is NULL");
    const bool need_x = dA != nullptr || (dB != nullptr && T_saved == nullptr);
    if (need_x && !X) return fail(NF4_ERR_INVALID_ARG, "X is NULL but dA, or dB without T_saved, is requested");
    if (!aligned16(dY) || (X && !aligned16(X)) || (T_saved && !aligned16(T_saved)) || (dX && !aligned16(dX)) ||
        (dA && !aligned16(dA)) || (dB && !aligned16(dB)))
        return fail(NF4_ERR_MISALIGNED, "an array argument is not 16-byte aligned");
    if (!dX && !dA && !dB) return ok();
    rc = check_ws(ws, ws_bytes, bwd_workspace_bytes(M, w->d_out, w->d_in, r, kPlanSMs));
    if (rc) return rc;
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    LayerCtx c{w->codes, w->qscale, w->scale2, w->scale_mean, w->absmax, w->d_out, w->d_in, kPlanSMs,
               static_cast<cudaStream_t>(stream)};
    rc = layer_bwd(c, A, B, r, scaling, X, T_saved, dY, M, dX, dA, dB, accumulate_grads,
                   static_cast<uint8_t*>(ws));
    if (rc == -1) return fail(NF4_ERR_CUDA, "qlora_linear_bwd: tensor map encoding failed");
    if (rc) return fail(NF4_ERR_CUDA, "qlora_linear_bwd launch: %s", cudaGetErrorString(layer_last_cuda_error()));
    return ok();
}

const char* nf4lora_last_error_string(void) { return t_last_error.c_str(); }

size_t nf4_merge_workspace_bytes(int64_t d_out, int64_t d_in) {
    if (!valid_weight_shape(d_out, d_in)) return 0;
    return static_cast<size_t>(align256(d_out * d_in * 4) + quant_ws_bytes(d_out, d_in));
}

static int check_merge_args(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling) {
    int rc = check_tensor(w);
    if (rc) return rc;
    if (r < 1 || r > 256) return fail(NF4_ERR_INVALID_ARG, "r = %d outside [1, 256]", r);
    if (!std::isfinite(scaling)) return fail(NF4_ERR_INVALID_ARG, "scaling is not finite");
    if (!A || !B) return fail(NF4_ERR_INVALID_ARG, "A or B is NULL");
    if (!aligned16(A) || !aligned16(B)) return fail(NF4_ERR_MISALIGNED, "A or B not 16-byte aligned");
    return NF4_OK;
}

int nf4_merge_lora(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling, float* W_merged,
                   void* stream) {
    int rc = check_merge_args(w, A, B, r, scaling);
    if (rc) return rc;
    if (W_merged == nullptr) return fail(NF4_ERR_INVALID_ARG, "W_merged is NULL");
    if (!aligned16(W_merged)) return fail(NF4_ERR_MISALIGNED, "W_merged not 16-byte aligned");
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    const cudaError_t e = launch_merge_lora(w->codes, w->qscale, w->scale2, w->scale_mean, w->absmax, A, B, r,
                                            w->d_out, w->d_in, scaling, W_merged, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_merge_lora launch: %s", cudaGetErrorString(e));
    return ok();
}

int nf4_merge_requantize(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling,
                         const nf4_tensor* out, void* ws, size_t ws_bytes, void* stream) {
    int rc = check_merge_args(w, A, B, r, scaling);
    if (rc) return rc;
    rc = check_tensor(out);
    if (rc) return rc;
    if (out->d_out != w->d_out || out->d_in != w->d_in)
        return fail(NF4_ERR_INVALID_ARG, "out describes [%lld, %lld], the weight is [%lld, %lld]",
                    (long long)out->d_out, (long long)out->d_in, (long long)w->d_out, (long long)w->d_in);
    const int64_t n = w->d_out * w->d_in;
    rc = check_ws(ws, ws_bytes, align256(n * 4) + quant_ws_bytes(w->d_out, w->d_in));
    if (rc) return rc;
    int sms = 0;
    rc = check_device(&sms);
    if (rc) return rc;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    float* merged = reinterpret_cast<float*>(w8);
    float* absmax = reinterpret_cast<float*>(w8 + align256(n * 4));
    double* tile_sums = reinterpret_cast<double*>(w8 + align256(n * 4) + align256(n / 64 * 4));
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_merge_lora(w->codes, w->qscale, w->scale2, w->scale_mean, w->absmax, A, B, r, w->d_out,
                                      w->d_in, scaling, merged, st);
    if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_merge_requantize launch: %s", cudaGetErrorString(e));
    // the merged weight is complete before the encoder starts (an ordinary
    // launch), so `out` may be `w` itself
    if (out->absmax != nullptr)
        e = launch_nf4_quantize(merged, n, out->codes, nullptr, nullptr, nullptr, out->absmax, nullptr, sms, st);
    else
        e = launch_nf4_quantize(merged, n, out->codes, out->qscale, out->scale2, out->scale_mean, absmax, tile_sums,
                                sms, st);
    if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "nf4_merge_requantize launch: %s", cudaGetErrorString(e));
    return ok();
}

int lora_adamw_step(const lora_adamw_tensor* tensors, int count, const lora_adamw_hparams* h, void* stream) {
    if (tensors == nullptr || h == nullptr) return fail(NF4_ERR_INVALID_ARG, "tensors or hparams is NULL");
    if (count < 1 || count > 1024) return fail(NF4_ERR_INVALID_ARG, "count %d outside [1, 1024]", count);
    const double lr = h->lr, b1 = h->beta1, b2 = h->beta2, eps = h->eps, wd = h->weight_decay;
    if (!(std::isfinite(lr) && lr >= 0.0) || !(b1 >= 0.0 && b1 < 1.0) || !(b2 >= 0.0 && b2 < 1.0) ||
        !(std::isfinite(eps) && eps > 0.0) || !(std::isfinite(wd) && wd >= 0.0) || h->step < 1)
        return fail(NF4_ERR_INVALID_ARG, "hyper-parameters out of range (lr >= 0, 0 <= beta < 1, eps > 0, "
                                         "weight_decay >= 0, step >= 1)");
    for (int i = 0; i < count; ++i) {
        const lora_adamw_tensor& t = tensors[i];
        if (t.n < 0) return fail(NF4_ERR_INVALID_ARG, "tensor %d: n < 0", i);
        if (t.n == 0) continue;
        if (!t.master || !t.grad || !t.m || !t.v) return fail(NF4_ERR_INVALID_ARG, "tensor %d: NULL pointer", i);
        if (!aligned16(t.master) || !aligned16(t.grad) || !aligned16(t.m) || !aligned16(t.v) ||
            (t.param && !aligned16(t.param)))
            return fail(NF4_ERR_MISALIGNED, "tensor %d: pointer not 16-byte aligned", i);
    }
    int sms = 0;
    int rc = check_device(&sms);
    if (rc) return rc;
    const double t = static_cast<double>(h->step);
    AdamwConsts c;
    c.decay = static_cast<float>(1.0 - lr * wd);
    c.b1 = h->beta1;
    c.omb1 = static_cast<float>(1.0 - b1);
    c.b2 = h->beta2;
    c.omb2 = static_cast<float>(1.0 - b2);
    c.step_size = static_cast<float>(lr / (1.0 - std::pow(b1, t)));
    c.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(b2, t)));
    c.eps = h->eps;
    for (int i0 = 0; i0 < count; i0 += kAdamwMaxTensors) {
        AdamwBatch b{};
        for (int i = i0; i < count && b.count < kAdamwMaxTensors; ++i) {
            const lora_adamw_tensor& src = tensors[i];
            const int k = b.count++;
            b.p[k] = src.master;
            b.p16[k] = src.param;
            b.g[k] = src.grad;
            b.m[k] = src.m;
            b.v[k] = src.v;
            b.n[k] = src.n;
        }
        const cudaError_t e = launch_adamw(b, c, sms, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return fail(NF4_ERR_CUDA, "lora_adamw_step launch: %s", cudaGetErrorString(e));
    }
    return ok();
}

int nf4lora_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return fail(NF4_ERR_CUDA, "stream synchronisation failed: %s", cudaGetErrorString(cudaGetLastError()));
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return fail(NF4_ERR_CUDA, "status word access failed");
    if (v != 0) return fail(NF4_ERR_TIMEOUT, "a kernel abandoned a bounded wait (status %d)", v);
    return ok();
}

int nf4lora_debug_site(void* stream, unsigned int* site) {
    if (site == nullptr) return fail(NF4_ERR_INVALID_ARG, "site is NULL");
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return fail(NF4_ERR_CUDA, "stream synchronisation failed: %s", cudaGetErrorString(cudaGetLastError()));
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_debug_site, sizeof(v)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_debug_site, &zero, sizeof(zero)) != cudaSuccess)
        return fail(NF4_ERR_CUDA, "debug word access failed");
    *site = v;
    return ok();
}

int nf4lora_debug_build(void) {
#ifdef NF4LORA_DEBUG
    return 1;
#else
    return 0;
#endif
}

const char* nf4lora_version(void) {
#ifdef NF4LORA_DEBUG
    return "nf4lora 0.2.0 sm_100a debug";
#else
    return "nf4lora 0.2.0 sm_100a";
#endif
}

}  // extern "C"
