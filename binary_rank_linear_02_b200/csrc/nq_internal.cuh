// nq_internal.cuh -- shared internals of libnq (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "nq.h"

namespace nq {

// ---------------------------------------------------------------- workspace
// One per device.  Decode keeps t (batch x r fp32), the split partials of stage 1 and a
// per-row-group arrival counter; prefill keeps x' (batch x n fp16) and T (batch x r
// fp16); host-memory x / y are staged through xstage / ystage.
struct Workspace {
    int device = -1;
    size_t bytes = 0;
    char* base = nullptr;
    // carved regions
    float* t = nullptr;            // [8][r_cap] (decode)
    float* tgmax = nullptr;        // [8][r_cap/128] max |t| per 128-row group (decode)
    float* partials = nullptr;     // [split_cap][8][r_cap]
    int* counters = nullptr;       // [r_cap/128], zero between calls
    unsigned* status = nullptr;    // device status word(s)
    uint16_t* xprime = nullptr;    // [batch_cap][n_cap] fp16 (prefill)
    uint16_t* T = nullptr;         // [batch_cap][r_cap] fp16 (prefill)
    void* xstage = nullptr;        // staged host x
    float* ystage = nullptr;       // staged host y
    size_t xstage_bytes = 0, ystage_bytes = 0;
    int64_t r_cap = 0, n_cap = 0, m_cap = 0, batch_cap = 0, split_cap = 0;
};

// Returns the current device's workspace, grown to fit (m, n, r, batch).  nullptr on
// allocation failure (status set to NQ_ERR_NOMEM / NQ_ERR_CUDA).
Workspace* workspace_for(int64_t m, int64_t n, int64_t r, int64_t batch, int* status);

int sm_count();

// ---------------------------------------------------------------- launch helpers
// Launch a kernel with programmatic stream serialisation allowed, so that it may start
// while the previous kernel on the stream drains; it must call pdl_wait() before
// reading anything that kernel produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- entry points of the kernels
int decode_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                   const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                   Workspace* ws, cudaStream_t stream);

int prefill_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                    const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                    Workspace* ws, cudaStream_t stream);

int pack_device(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* out, unsigned* flag,
                cudaStream_t stream);
int unpack_device(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* out, cudaStream_t stream);

}  // namespace nq
