// rowwise_kernels.cuh -- the two bandwidth-bound kernels of the library:
//
//   row softmax   y_j = exp(x_j - max x) / sum_k exp(x_k - max x) per row
//                 (TileLang GPU kernel design article, paragraph 5: a row-wise
//                 softmax with max and sum reductions kept in registers)
//   vector add    C[i] = A[i] + B[i] in float32 (the same article, paragraph
//                 3, and the blog retelling's Step 3)
//
// Both read each input once and write each output once; their roofline is
// HBM bandwidth.  16-byte vector accesses when the rows / arrays allow them,
// element accesses otherwise; grids are sized in multiples of the SM count.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100.cuh"

namespace tl {

template <int DT>
__device__ __forceinline__ float half_to_float(uint16_t b)
{
    if constexpr (DT == 1)
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    else
        return __half2float(__ushort_as_half(b));
}

template <int DT>
__device__ __forceinline__ uint16_t float_to_half(float f)
{
    if constexpr (DT == 1)
        return __bfloat16_as_ushort(__float2bfloat16_rn(f));
    else
        return __half_as_ushort(__float2half_rn(f));
}

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ row softmax, one warp per row
// Rows of up to 32 * PER_LANE values live in registers: one read, one write.
template <int DT, int PER_LANE, bool VEC>
__global__ void __launch_bounds__(256) softmax_rows_warp_kernel(const uint16_t *__restrict__ X,
                                                                uint16_t *__restrict__ Y, int64_t rows, int cols)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
         row += warps_total) {
        const uint16_t *x = X + row * cols;
        uint16_t *y = Y + row * cols;
        float v[PER_LANE];
        float m = -INFINITY;
        if constexpr (VEC) {
            // lane reads 8 consecutive values per step; a step covers 256 columns
#pragma unroll
            for (int s = 0; s < PER_LANE / 8; ++s) {
                const int c = s * 256 + lane * 8;
                if (c < cols) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + c));
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        v[8 * s + 2 * h] = half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu));
                        v[8 * s + 2 * h + 1] = half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v[8 * s + e] = -INFINITY;
                }
            }
        } else {
#pragma unroll
            for (int s = 0; s < PER_LANE; ++s) {
                const int c = s * 32 + lane;
                v[s] = c < cols ? half_to_float<DT>(x[c]) : -INFINITY;
            }
        }
#pragma unroll
        for (int s = 0; s < PER_LANE; ++s)
            m = fmaxf(m, v[s]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float mb = m * kLog2e;
        float sum = 0.0f;
#pragma unroll
        for (int s = 0; s < PER_LANE; ++s) {
            v[s] = exp2_approx(fmaf(v[s], kLog2e, -mb));  // -inf (padding) -> 0
            sum += v[s];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float inv = 1.0f / sum;
        if constexpr (VEC) {
#pragma unroll
            for (int s = 0; s < PER_LANE / 8; ++s) {
                const int c = s * 256 + lane * 8;
                if (c < cols) {
                    uint4 w;
                    w.x = float_to_half<DT>(v[8 * s] * inv) | (static_cast<uint32_t>(float_to_half<DT>(v[8 * s + 1] * inv)) << 16);
                    w.y = float_to_half<DT>(v[8 * s + 2] * inv) | (static_cast<uint32_t>(float_to_half<DT>(v[8 * s + 3] * inv)) << 16);
                    w.z = float_to_half<DT>(v[8 * s + 4] * inv) | (static_cast<uint32_t>(float_to_half<DT>(v[8 * s + 5] * inv)) << 16);
                    w.w = float_to_half<DT>(v[8 * s + 6] * inv) | (static_cast<uint32_t>(float_to_half<DT>(v[8 * s + 7] * inv)) << 16);
                    *reinterpret_cast<uint4 *>(y + c) = w;
                }
            }
        } else {
#pragma unroll
            for (int s = 0; s < PER_LANE; ++s) {
                const int c = s * 32 + lane;
                if (c < cols)
                    y[c] = float_to_half<DT>(v[s] * inv);
            }
        }
    }
}

// ------------------------------------------------------------------ row softmax, one CTA per row, in registers
// Rows of up to THREADS * PER_THREAD values (16-byte aligned, a multiple of 8
// long) are read once into registers; block reductions through shared memory.
template <int DT, int PER_THREAD>
__global__ void __launch_bounds__(512) softmax_rows_cta_regs_kernel(const uint16_t *__restrict__ X,
                                                                    uint16_t *__restrict__ Y, int64_t rows, int cols)
{
    __shared__ float red[16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int step = blockDim.x * 8;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const uint16_t *x = X + row * cols;
        uint16_t *y = Y + row * cols;
        float v[PER_THREAD];
        float m = -INFINITY;
#pragma unroll
        for (int s = 0; s < PER_THREAD / 8; ++s) {
            const int c = s * step + tid * 8;
            if (c < cols) {
                const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + c));
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    v[8 * s + 2 * h] = half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu));
                    v[8 * s + 2 * h + 1] = half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[8 * s + e] = -INFINITY;
            }
        }
#pragma unroll
        for (int i = 0; i < PER_THREAD; ++i)
            m = fmaxf(m, v[i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0)
            red[warp] = m;
        __syncthreads();
        m = red[0];
        for (int w = 1; w < nwarps; ++w)
            m = fmaxf(m, red[w]);
        __syncthreads();
        const float mb = m * kLog2e;
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < PER_THREAD; ++i) {
            v[i] = exp2_approx(fmaf(v[i], kLog2e, -mb));
            sum += v[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0)
            red[warp] = sum;
        __syncthreads();
        sum = 0.0f;
        for (int w = 0; w < nwarps; ++w)
            sum += red[w];
        __syncthreads();
        const float inv = 1.0f / sum;
#pragma unroll
        for (int s = 0; s < PER_THREAD / 8; ++s) {
            const int c = s * step + tid * 8;
            if (c < cols) {
                uint32_t o[4];
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    o[h] = float_to_half<DT>(v[8 * s + 2 * h] * inv) |
                           (static_cast<uint32_t>(float_to_half<DT>(v[8 * s + 2 * h + 1] * inv)) << 16);
                *reinterpret_cast<uint4 *>(y + c) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// ------------------------------------------------------------------ row softmax, one CTA per row
// Any row length: pass 1 keeps a running (max, sum) per thread and merges
// them across the block; pass 2 reads the row again (from L2 for rows of up
// to a few hundred kilobytes) and writes y.
template <int DT>
__global__ void __launch_bounds__(512) softmax_rows_block_kernel(const uint16_t *__restrict__ X,
                                                                 uint16_t *__restrict__ Y, int64_t rows, int64_t cols,
                                                                 int peel)
{
    __shared__ float red_m[16], red_s[16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const uint16_t *x = X + row * cols;
        uint16_t *y = Y + row * cols;
        // split the row into a head (up to 7 values before the first 16-byte
        // boundary), a body of 8-value vectors and a tail; without `peel` (x
        // and y differently aligned) everything is handled value by value
        int64_t head = 0, nvec = 0;
        if (peel) {
            head = ((16 - (reinterpret_cast<uintptr_t>(x) & 15)) & 15) >> 1;
            if (head > cols)
                head = cols;
            nvec = (cols - head) >> 3;
        }
        const int64_t body_end = head + (nvec << 3);
        float m = -INFINITY, s = 0.0f;  // in log2 units: s = sum 2^(t - m)
        auto absorb = [&](float t) {
            if (t > m) {
                s = s * exp2_approx(m - t) + 1.0f;
                m = t;
            } else {
                s += exp2_approx(t - m);
            }
        };
        for (int64_t c = tid; c < head; c += blockDim.x)
            absorb(half_to_float<DT>(x[c]) * kLog2e);
        for (int64_t i = tid; i < nvec; i += blockDim.x) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + head) + i);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            float t[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                t[2 * h] = half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu)) * kLog2e;
                t[2 * h + 1] = half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16)) * kLog2e;
            }
            float mx = t[0];
#pragma unroll
            for (int e = 1; e < 8; ++e)
                mx = fmaxf(mx, t[e]);
            if (mx > m) {
                s = (m == -INFINITY) ? 0.0f : s * exp2_approx(m - mx);
                m = mx;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e)
                s += exp2_approx(t[e] - m);
        }
        for (int64_t c = body_end + tid; c < cols; c += blockDim.x)
            absorb(half_to_float<DT>(x[c]) * kLog2e);
        // merge (m, s) across the warp, then across warps
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
            const float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.0f : s * exp2_approx(m - mm)) + (m2 == -INFINITY ? 0.0f : s2 * exp2_approx(m2 - mm));
            m = mm;
        }
        if (lane == 0) {
            red_m[warp] = m;
            red_s[warp] = s;
        }
        __syncthreads();
        float M = -INFINITY;
        for (int w = 0; w < nwarps; ++w)
            M = fmaxf(M, red_m[w]);
        float S = 0.0f;
        for (int w = 0; w < nwarps; ++w)
            if (red_m[w] != -INFINITY)
                S += red_s[w] * exp2_approx(red_m[w] - M);
        __syncthreads();  // red_* reused by the next row
        const float inv = 1.0f / S;
        for (int64_t c = tid; c < head; c += blockDim.x)
            y[c] = float_to_half<DT>(exp2_approx(fmaf(half_to_float<DT>(x[c]), kLog2e, -M)) * inv);
        for (int64_t i = tid; i < nvec; i += blockDim.x) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + head) + i);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float a = exp2_approx(fmaf(half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu)), kLog2e, -M)) * inv;
                const float b = exp2_approx(fmaf(half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16)), kLog2e, -M)) * inv;
                o[h] = float_to_half<DT>(a) | (static_cast<uint32_t>(float_to_half<DT>(b)) << 16);
            }
            reinterpret_cast<uint4 *>(y + head)[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        for (int64_t c = body_end + tid; c < cols; c += blockDim.x)
            y[c] = float_to_half<DT>(exp2_approx(fmaf(half_to_float<DT>(x[c]), kLog2e, -M)) * inv);
    }
}

// ------------------------------------------------------------------ vector add
__global__ void __launch_bounds__(256) vector_add_kernel(const float *__restrict__ A, const float *__restrict__ B,
                                                         float *__restrict__ C, int64_t n, int vec)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    if (vec) {
        const int64_t n4 = n >> 2;
        const float4 *a4 = reinterpret_cast<const float4 *>(A);
        const float4 *b4 = reinterpret_cast<const float4 *>(B);
        float4 *c4 = reinterpret_cast<float4 *>(C);
        int64_t i = t;
        for (; i + 3 * stride < n4; i += 4 * stride) {  // four vectors in flight per thread
            float4 a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = __ldcs(a4 + i + u * stride);
                b[u] = __ldcs(b4 + i + u * stride);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                __stcs(c4 + i + u * stride, make_float4(a[u].x + b[u].x, a[u].y + b[u].y, a[u].z + b[u].z, a[u].w + b[u].w));
        }
        for (; i < n4; i += stride) {
            const float4 a = __ldcs(a4 + i), b = __ldcs(b4 + i);
            __stcs(c4 + i, make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w));
        }
        for (int64_t i = (n4 << 2) + t; i < n; i += stride)
            C[i] = A[i] + B[i];
    } else {
        for (int64_t i = t; i < n; i += stride)
            C[i] = A[i] + B[i];
    }
}

} // namespace tl
