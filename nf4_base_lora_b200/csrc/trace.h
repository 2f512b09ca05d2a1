// Launch tracing: while enabled, every kernel the library launches is
// bracketed by two CUDA events recorded on its stream.  Inside a stream
// capture the records become event-record nodes of the graph (recorded with
// the external flag), so each replay records them again.
#pragma once

#include <cuda_runtime.h>

namespace nf4lora {

// Returns a slot id, or -1 when tracing is off or the record pool is full.
int trace_begin(const char* name, cudaStream_t stream);
void trace_end(int slot, cudaStream_t stream);

struct TraceScope {
    int slot;
    cudaStream_t stream;
    TraceScope(const char* name, cudaStream_t s) : slot(trace_begin(name, s)), stream(s) {}
    ~TraceScope() { trace_end(slot, stream); }
};

}  // namespace nf4lora
