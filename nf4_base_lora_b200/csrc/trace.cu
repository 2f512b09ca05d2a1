// Launch tracing for the library's own kernels (see trace.h), exported through
// the nf4lora_trace_* entry points of the C ABI.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "nf4lora.h"
#include "trace.h"

namespace nf4lora {

namespace {

struct Record {
    std::string name;
    cudaEvent_t start = nullptr, stop = nullptr;
};

std::mutex g_mu;
std::atomic<bool> g_on{false};
std::vector<Record> g_pool;
int g_used = 0;
int g_count = 0;

void destroy_pool() {
    for (auto& r : g_pool) {
        if (r.start) cudaEventDestroy(r.start);
        if (r.stop) cudaEventDestroy(r.stop);
    }
    g_pool.clear();
    g_used = 0;
}

// Inside a stream capture a plain record only marks a point for the capture's
// own dependency tracking; the external flag makes it an event-record node of
// the graph, which records the event at every replay.
void record(cudaEvent_t ev, cudaStream_t stream) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, stream);
}

}  // namespace

int trace_begin(const char* name, cudaStream_t stream) {
    if (!g_on.load(std::memory_order_relaxed)) return -1;
    std::lock_guard<std::mutex> lk(g_mu);
    ++g_count;
    if (g_used >= static_cast<int>(g_pool.size())) return -1;
    const int slot = g_used++;
    g_pool[slot].name = name;
    record(g_pool[slot].start, stream);
    return slot;
}

void trace_end(int slot, cudaStream_t stream) {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (slot < static_cast<int>(g_pool.size())) record(g_pool[slot].stop, stream);
}

}  // namespace nf4lora

using namespace nf4lora;

extern "C" {

int nf4lora_trace_start(int max_launches) {
    if (max_launches < 0 || max_launches > (1 << 20)) return NF4_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    destroy_pool();
    g_pool.resize(static_cast<size_t>(max_launches));
    for (auto& r : g_pool) {
        if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) {
            destroy_pool();
            return NF4_ERR_CUDA;
        }
    }
    g_count = 0;
    g_on.store(true);
    return NF4_OK;
}

int nf4lora_trace_stop(void) {
    g_on.store(false);
    return NF4_OK;
}

int nf4lora_trace_count(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_count;
}

int nf4lora_trace_get(int i, char* name, size_t name_len, float* ms) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (i < 0 || i >= g_used) return NF4_ERR_INVALID_ARG;
    if (name != nullptr && name_len > 0) {
        std::strncpy(name, g_pool[i].name.c_str(), name_len - 1);
        name[name_len - 1] = '\0';
    }
    if (ms != nullptr) {
        if (cudaEventSynchronize(g_pool[i].stop) != cudaSuccess ||
            cudaEventElapsedTime(ms, g_pool[i].start, g_pool[i].stop) != cudaSuccess) {
            cudaGetLastError();  // the failure is reported through the return value
            return NF4_ERR_CUDA;
        }
    }
    return NF4_OK;
}

}  // extern "C"
