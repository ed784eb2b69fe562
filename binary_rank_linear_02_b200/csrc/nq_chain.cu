// nq_chain.cu -- the two small element-wise steps between the factorised layers of a
// decode chain: rounding a layer's fp32 output to the bfloat16 input of the next layer,
// and re-normalising a block's output to unit root-mean-square before the next block.
//
// A decoder runs its quantised linear layers one after the other (hardwired.dev,
// "NanoQuant jednoduse: 70B model na herni grafice", section "Cisla": decode tokens/s of
// a whole quantised 70B model).  The pages print neither what sits between the layers
// nor any normalisation; these two kernels are the library's helpers for chaining its
// own forward calls (each layer takes bfloat16 x and returns fp32 y).
//
// Both kernels are memory-trivial (tens of KB per call at decode sizes) and sit on the
// chain's critical path, so they are shaped for latency: launched with programmatic
// dependent launch, they let the next kernel start its weight prefetch early and read
// their input only after the producing kernel has finished.
//
// Also here: the gather of pinned host inputs, and the per-column dot products over the
// tokens that finish the scale gradients of the backward pass.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nq_internal.cuh"

namespace nq {
namespace {

constexpr int kCastThreads = 256;
constexpr int kNormThreads = 512;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// dst[i] = bf16(src[i]) (round to nearest, ties to even); 8 elements per thread step.
__global__ void __launch_bounds__(kCastThreads) cast_kernel(const float* __restrict__ src, int64_t count,
                                                            uint16_t* __restrict__ dst) {
    pdl_wait();
    pdl_trigger();
    const int64_t groups = count / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups; g += stride) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(src) + 2 * g);
        const float4 b = __ldcg(reinterpret_cast<const float4*>(src) + 2 * g + 1);
        reinterpret_cast<uint4*>(dst)[g] =
            make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    }
    for (int64_t i = groups * 8 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += stride)
        dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldcg(src + i)));
}

// One CTA per row: dst[row][j] = bf16(src[row][j] * (1 / sqrt(sum_j src^2 / cols))).
// A row whose sum of squares is 0 is rounded as it is (signed zeros kept).
__global__ void __launch_bounds__(kNormThreads, 1) rms_norm_kernel(const float* __restrict__ src, int64_t cols,
                                                                uint16_t* __restrict__ dst) {
    __shared__ float warp_sums[kNormThreads / 32];
    __shared__ float inv_rms;
    pdl_wait();
    pdl_trigger();
    const float* row = src + (int64_t)blockIdx.x * cols;
    uint16_t* out = dst + (int64_t)blockIdx.x * cols;
    const bool vec = (cols % 8) == 0;  // rows then start on 32-byte (src) and 16-byte (dst) boundaries
    float ss = 0.f;
    if (vec) {
        for (int64_t g = threadIdx.x; g < cols / 4; g += blockDim.x) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(row) + g);
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        }
    } else {
        for (int64_t j = threadIdx.x; j < cols; j += blockDim.x) {
            const float v = __ldcg(row + j);
            ss = fmaf(v, v, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float s = threadIdx.x < (blockDim.x >> 5) ? warp_sums[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) inv_rms = s > 0.f ? 1.0f / sqrtf(s / (float)cols) : 1.0f;
    }
    __syncthreads();
    const float k = inv_rms;
    if (vec) {
        for (int64_t g = threadIdx.x; g < cols / 8; g += blockDim.x) {
            const float4 a = __ldcg(reinterpret_cast<const float4*>(row) + 2 * g);
            const float4 b = __ldcg(reinterpret_cast<const float4*>(row) + 2 * g + 1);
            reinterpret_cast<uint4*>(out)[g] = make_uint4(pack_bf16x2(a.x * k, a.y * k), pack_bf16x2(a.z * k, a.w * k),
                                                          pack_bf16x2(b.x * k, b.y * k), pack_bf16x2(b.z * k, b.w * k));
        }
    } else {
        for (int64_t j = threadIdx.x; j < cols; j += blockDim.x)
            out[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldcg(row + j) * k));
    }
}

// Copies up to kMaxGather buffers (16-byte multiples, 16-byte aligned), one per grid row;
// used to bring the x of a call from pinned host memory (read through its device
// address) into the device staging buffer in one launch instead of one copy per layer.
__global__ void __launch_bounds__(256) gather_kernel(const __grid_constant__ GatherList list) {
    pdl_trigger();  // the decode kernels may launch and stage their weights during the copy
    if ((int)blockIdx.y >= list.count) return;
    const GatherSeg& g = list.seg[blockIdx.y];
    const uint4* src = static_cast<const uint4*>(g.src);
    uint4* dst = static_cast<uint4*>(g.dst);
    const int64_t n = (int64_t)(g.bytes / 16);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

// Scale gradients: out[i] = sum_b bf16(a[b][i]) * z[b][i], one thread per i, the tokens in
// increasing order (deterministic).  z comes from the kernel before (programmatic wait).
// out[i] = sum_b bf16(a[b][i]) * z[b][i]: the tokens in chunks of kDotChunk, chunk c's sum
// (tokens in order) into part[c][i] by CTA row c, or straight into out when there is one
// chunk; then col_sum_kernel adds the chunks' sums in chunk order (a fixed order).
constexpr int64_t kDotChunk = 64;

__global__ void __launch_bounds__(256) col_dot_kernel(const uint16_t* __restrict__ a, const float* __restrict__ z,
                                                      int64_t batch, int64_t len, float* __restrict__ part) {
    pdl_wait();
    pdl_trigger();
    const int64_t b0 = (int64_t)blockIdx.y * kDotChunk;
    const int64_t b1 = b0 + kDotChunk < batch ? b0 + kDotChunk : batch;
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= len) return;
    float acc = 0.f;
    for (int64_t b = b0; b < b1; ++b) acc = fmaf(__uint_as_float((uint32_t)a[b * len + i] << 16), z[b * len + i], acc);
    part[(int64_t)blockIdx.y * len + i] = acc;
}

__global__ void __launch_bounds__(256) col_sum_kernel(const float* __restrict__ part, int64_t chunks, int64_t len,
                                                      float* __restrict__ out) {
    pdl_wait();
    pdl_trigger();
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= len) return;
    float acc = 0.f;
    for (int64_t c = 0; c < chunks; ++c) acc += __ldcg(part + c * len + i);
    out[i] = acc;
}

__global__ void fill_u16_kernel(uint16_t* p, int64_t count, uint16_t value) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = value;
}

// The straight-through gradients of the factors: out[i][k] = s[i] * sum_b a[b][i] * t[b][k]
// (a bf16 batch x M, t fp32 batch x R).  A 16 x 16 thread block computes a 64 x 64 tile,
// four by four outputs per thread, staging 32 tokens of a and t at a time in shared
// memory; the tokens are added in order (deterministic).
constexpr int kOuterTile = 64, kOuterTokens = 32;

__global__ void __launch_bounds__(256) outer_kernel(const uint16_t* __restrict__ a, const uint16_t* __restrict__ s,
                                                    const float* __restrict__ t, int64_t batch, int64_t M, int64_t R,
                                                    float* __restrict__ out) {
    __shared__ float as[kOuterTokens][kOuterTile];
    __shared__ float ts[kOuterTokens][kOuterTile];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int64_t i0 = (int64_t)blockIdx.y * kOuterTile, k0 = (int64_t)blockIdx.x * kOuterTile;
    float acc[4][4] = {};
    for (int64_t b0 = 0; b0 < batch; b0 += kOuterTokens) {
        for (int e = threadIdx.x; e < kOuterTokens * kOuterTile; e += 256) {
            const int bb = e / kOuterTile, c = e % kOuterTile;
            const int64_t b = b0 + bb;
            as[bb][c] = (b < batch && i0 + c < M) ? __uint_as_float((uint32_t)a[b * M + i0 + c] << 16) : 0.f;
            ts[bb][c] = (b < batch && k0 + c < R) ? t[b * R + k0 + c] : 0.f;
        }
        __syncthreads();
        for (int bb = 0; bb < kOuterTokens; ++bb) {
            float av[4], tv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                av[q] = as[bb][ty + 16 * q];
                tv[q] = ts[bb][tx + 16 * q];
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(av[p], tv[q], acc[p][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int64_t i = i0 + ty + 16 * p;
        if (i >= M) continue;
        const float si = __half2float(__ushort_as_half(s[i]));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t k = k0 + tx + 16 * q;
            if (k < R) out[i * R + k] = si * acc[p][q];
        }
    }
}

}  // namespace

int gather_device(const GatherList& list, cudaStream_t stream) {
    if (list.count <= 0) return NQ_OK;
    size_t most = 0;
    for (int i = 0; i < list.count; ++i) most = list.seg[i].bytes > most ? list.seg[i].bytes : most;
    int gx = (int)((most / 16 + 255) / 256);
    if (gx < 1) gx = 1;
    if (gx > 32) gx = 32;
    gather_kernel<<<dim3((unsigned)gx, (unsigned)list.count), 256, 0, stream>>>(list);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

// The rank-l envelope's sum: y[e] += terms[q][e] for q = 0 .. nterms-1 in that order
// (y holds the first term), four elements per thread step.
__global__ void __launch_bounds__(256) envelope_sum_kernel(float* __restrict__ y, const float* __restrict__ terms,
                                                           int nterms, int64_t count) {
    pdl_wait();
    pdl_trigger();
    const int64_t groups = count / 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups; g += stride) {
        float4 acc = __ldcg(reinterpret_cast<const float4*>(y) + g);
        for (int q = 0; q < nterms; ++q) {
            const float4 t = __ldcg(reinterpret_cast<const float4*>(terms + (int64_t)q * count) + g);
            acc.x += t.x;
            acc.y += t.y;
            acc.z += t.z;
            acc.w += t.w;
        }
        reinterpret_cast<float4*>(y)[g] = acc;
    }
    for (int64_t i = groups * 4 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += stride) {
        float acc = __ldcg(y + i);
        for (int q = 0; q < nterms; ++q) acc += __ldcg(terms + (int64_t)q * count + i);
        y[i] = acc;
    }
}

int cast_f32_bf16_device(const float* src, int64_t count, uint16_t* dst, cudaStream_t stream) {
    int64_t blocks = (count / 8 + kCastThreads - 1) / kCastThreads;
    if (blocks < 1) blocks = 1;
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    return launch_pdl(cast_kernel, dim3((unsigned)blocks), dim3(kCastThreads), 0, stream, src, count, dst) ==
                   cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

int rms_normalize_bf16_device(const float* src, int64_t rows, int64_t cols, uint16_t* dst, cudaStream_t stream) {
    return launch_pdl(rms_norm_kernel, dim3((unsigned)rows), dim3(kNormThreads), 0, stream, src, cols, dst) ==
                   cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

int64_t col_dot_scratch_floats(int64_t batch, int64_t len) {
    const int64_t chunks = (batch + kDotChunk - 1) / kDotChunk;
    return chunks > 1 ? chunks * len : 0;
}

int col_dot_device(const uint16_t* a, const float* z, int64_t batch, int64_t len, float* out, float* scratch,
                   cudaStream_t stream) {
    const int64_t chunks = (batch + kDotChunk - 1) / kDotChunk;
    const dim3 grid((unsigned)((len + 255) / 256), (unsigned)chunks);
    if (chunks == 1)
        return launch_pdl(col_dot_kernel, grid, dim3(256), 0, stream, a, z, batch, len, out) == cudaSuccess
                   ? NQ_OK
                   : NQ_ERR_CUDA;
    if (launch_pdl(col_dot_kernel, grid, dim3(256), 0, stream, a, z, batch, len, scratch) != cudaSuccess)
        return NQ_ERR_CUDA;
    return launch_pdl(col_sum_kernel, dim3((unsigned)((len + 255) / 256)), dim3(256), 0, stream,
                      (const float*)scratch, chunks, len, out) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

int fill_u16_device(uint16_t* p, int64_t count, uint16_t value, cudaStream_t stream) {
    int64_t blocks = (count + 255) / 256;
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    if (blocks < 1) blocks = 1;
    fill_u16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p, count, value);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

int outer_device(const uint16_t* a, const uint16_t* s, const float* t, int64_t batch, int64_t M, int64_t R,
                 float* out, cudaStream_t stream) {
    const dim3 grid((unsigned)((R + kOuterTile - 1) / kOuterTile), (unsigned)((M + kOuterTile - 1) / kOuterTile));
    outer_kernel<<<grid, 256, 0, stream>>>(a, s, t, batch, M, R, out);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

int envelope_sum_device(float* y, const float* terms, int nterms, int64_t count, cudaStream_t stream) {
    int64_t blocks = (count / 4 + 255) / 256;
    if (blocks < 1) blocks = 1;
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    return launch_pdl(envelope_sum_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, y, terms, nterms, count) ==
                   cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

}  // namespace nq
