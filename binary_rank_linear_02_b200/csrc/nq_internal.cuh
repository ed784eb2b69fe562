// nq_internal.cuh -- shared internals of libnq (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "nq.h"

namespace nq {

constexpr int kMaxGroup = 16;         // layers per decode launch
constexpr int kDecodeMaxSplits = 64;  // stage-1 column splits per layer

// ---------------------------------------------------------------- workspace
// One per device.  Decode keeps t (batch x r fp32 per layer) and the max |t| of each
// 128-row block; prefill keeps x' (batch x n fp16) and T (batch x r fp16); both use
// `partials` and `counters` for split reductions; host-memory x go through xstage (pinned
// x by a gather kernel, pageable x by a copy) and pageable host y through ystage.
struct Workspace {
    int device = -1;
    size_t bytes = 0;
    char* base = nullptr;
    // carved regions
    float* t = nullptr;            // [t_cap] (decode: sum over a launch's layers of batch x r)
    float* tgmax = nullptr;        // [tgmax_cap] (decode: batch x r/128 per layer)
    float* partials = nullptr;     // [partial_cap] (stage-1 column splits; prefill K splits; norm sums)
    int* counters = nullptr;       // [counter_cap] (arrival counters, zero between calls)
    unsigned* status = nullptr;    // [0]: pack value check, [1]: device wait timeout
    uint16_t* xprime = nullptr;    // [batch_cap][n_cap] fp16 (prefill)
    uint16_t* T = nullptr;         // [batch_cap][r_cap] fp16 (prefill)
    float* xscale = nullptr;       // [batch_cap] (prefill: 2^e per token, the power of two x' and T carry)
    void* xstage = nullptr;        // staged host x
    float* ystage = nullptr;       // staged host y
    size_t xstage_bytes = 0, ystage_bytes = 0;
    uint16_t* ones = nullptr;      // [ones_count] fp16 1.0 (scale gradients: the layer without a scale)
    float* gstage = nullptr;       // scale gradients: batch x max(m, n) outputs of the layer without a scale
    size_t ones_count = 0, gstage_bytes = 0;
    float* env = nullptr;          // envelope terms 1 .. l-1: (l-1) x batch x m fp32
    size_t env_bytes = 0;
    void* dense = nullptr;         // factor gradients on the tensor cores: the split rank vectors
    size_t dense_bytes = 0;
    size_t t_cap = 0, tgmax_cap = 0, partial_cap = 0, counter_cap = 0;
    int64_t r_cap = 0, n_cap = 0, m_cap = 0, batch_cap = 0, rsum_cap = 0;
};

// What a decode launch needs from the workspace, in elements.
struct DecodeNeed {
    int64_t t = 0, tgmax = 0, partials = 0, counters = 0;
};

// Returns the current device's workspace, grown to fit a prefill layer of at most
// (m, n, r) and `batch` tokens and a decode launch needing `dec`.  nullptr on failure
// (status set to NQ_ERR_NOMEM / NQ_ERR_CUDA).
Workspace* workspace_for(int64_t m, int64_t n, int64_t r, int64_t batch, const DecodeNeed& dec, int* status);

// One factorised layer of a decode launch.
struct DecodeCall {
    const uint16_t* x;
    const uint32_t* Upk;
    const uint32_t* Vpk;
    const uint16_t* s1;
    const uint16_t* s2;
    float* y;
    int64_t m, n, r;
    uint16_t* y_bf16 = nullptr;  // optional: bf16(y), batch x m
    uint16_t* y_norm = nullptr;  // optional: bf16(y / rms(y)) per token, batch x m
};

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
int decode_forward_group(const DecodeCall* calls, int count, int64_t batch, Workspace* ws, cudaStream_t stream,
                         int max_splits = kDecodeMaxSplits, bool stage1_only = false);
// t = V^T (s2 (.) x) alone (batch x r fp32, any batch: the decode stage-1 kernel, up to
// NQ_DECODE_MAX_BATCH tokens per launch, each launch's t copied out of the workspace).
int decode_rank_vector(const uint16_t* x, const uint32_t* Vpk, const uint16_t* s2, int64_t n, int64_t r,
                       int64_t batch, float* t, Workspace* ws, cudaStream_t stream);
// t = V^T (s2 (.) x) (batch x r fp32) by the prefill kernels, for batch > NQ_DECODE_MAX_BATCH;
// ones: at least r fp16 1.0
int prefill_rank_vector(const uint16_t* x, const uint32_t* Vpk, const uint16_t* s2, int64_t n, int64_t r,
                        int64_t batch, float* t, const uint16_t* ones, Workspace* ws, cudaStream_t stream);
// out[i][k] = s[i] * sum_b bf16(a[b][i]) * t[b][k] (M x R fp32) on the tensor cores (M, R
// multiples of 128), t split into two bf16 halves; scratch of outer_tc_scratch_bytes.
int64_t outer_tc_scratch_bytes(int64_t batch, int64_t M, int64_t R);
int outer_tc(const uint16_t* a, const uint16_t* s, const float* t, int64_t batch, int64_t M, int64_t R, float* out,
             void* scratch, unsigned* status, cudaStream_t stream);
// out (M x R fp32) = Aop F + rho (D - E) on the tensor cores: Aop is M x K with A bfloat16
// given as M x K rows (a_kmajor_rows) or as K x M rows (Aop = A^T: read in place), K a
// multiple of 64; F is K x R fp32 split into three bfloat16 parts (scratch of
// dense_af_scratch_bytes); D and E laid out as out, rho a device scalar; M, R multiples of 128.
int64_t dense_af_scratch_bytes(int64_t K, int64_t R);
int dense_af(const uint16_t* A, bool a_kmajor_rows, int64_t M, int64_t K, const float* F, int64_t R, float* out,
             const float* D, const float* E, const float* rho, void* scratch, unsigned* status, cudaStream_t stream);
// out[i][k] = s[i] * sum over b (increasing) of bf16(a[b][i]) * t[b][k]: M x R fp32
int outer_device(const uint16_t* a, const uint16_t* s, const float* t, int64_t batch, int64_t M, int64_t R,
                 float* out, cudaStream_t stream);
void decode_workspace_need(const DecodeCall* calls, int count, int64_t batch, int max_splits, int64_t* t_floats,
                           int64_t* tgmax_floats, int64_t* partial_floats, int64_t* counter_ints);

int decode_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                   const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                   Workspace* ws, cudaStream_t stream);

// Scratch of the prefill path's split-K items (fp32 partial tiles and arrival counters).
void prefill_workspace_need(int64_t m, int64_t n, int64_t r, int64_t batch, int64_t* partial_floats,
                            int64_t* counter_ints);
// Runs the bounded device wait on a barrier nothing arrives on (failure-path self-test).
int selftest_wait_timeout(int64_t limit_ns, Workspace* ws, cudaStream_t stream);
int prefill_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                    const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                    Workspace* ws, cudaStream_t stream);

int pack_device(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* out, unsigned* flag,
                cudaStream_t stream);
int unpack_device(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* out, cudaStream_t stream);
int transpose_device(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out, cudaStream_t stream);
// out[i] = sum_b bf16(a[b][i]) * z[b][i], for i < len: chunks of 64 tokens summed in token
// order, then the chunks in order (deterministic); scratch of col_dot_scratch_floats floats
int64_t col_dot_scratch_floats(int64_t batch, int64_t len);
int col_dot_device(const uint16_t* a, const float* z, int64_t batch, int64_t len, float* out, float* scratch,
                   cudaStream_t stream);
int fill_u16_device(uint16_t* p, int64_t count, uint16_t value, cudaStream_t stream);
constexpr int kMaxGather = 16;
struct GatherSeg {
    const void* src;
    void* dst;
    size_t bytes;  // a multiple of 16
};
struct GatherList {
    GatherSeg seg[kMaxGather];
    int count;
};
int gather_device(const GatherList& list, cudaStream_t stream);
int cast_f32_bf16_device(const float* src, int64_t count, uint16_t* dst, cudaStream_t stream);
// y[e] += terms[q * count + e] for q = 0 .. nterms-1 in order (the envelope's sum)
int envelope_sum_device(float* y, const float* terms, int nterms, int64_t count, cudaStream_t stream);
int rms_normalize_bf16_device(const float* src, int64_t rows, int64_t cols, uint16_t* dst, cudaStream_t stream);

}  // namespace nq
