// rowwise_kernels.cuh -- the two bandwidth-bound kernels of the library:
//
//   row softmax   y_j = exp(x_j - max x) / sum_k exp(x_k - max x) per row
//                 (TileLang GPU kernel design article, paragraph 5: a row-wise
//                 softmax with max and sum reductions kept in registers)
//   vector add    C[i] = A[i] + B[i] in float32 (the same article, paragraph
//                 3, and the blog retelling's Step 3)
//
// Both read each input once and write each output once; their roofline is
// HBM bandwidth.  The softmax weights use the flush-to-zero 2^x (one MUFU
// op): a probability below 2^-126 (1.2e-38) comes out as 0.  16-byte vector accesses when the rows / arrays allow them,
// element accesses otherwise; grids are sized in multiples of the SM count.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100.cuh"
#include "gemm_kernel.cuh"  // the library's device error word (g_device_error)

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

// 8 16-bit values of one 16-byte word, widened to float
template <int DT>
__device__ __forceinline__ void unpack8(const uint4 &w, float *v)
{
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        v[2 * h] = half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu));
        v[2 * h + 1] = half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16));
    }
}

// 8 floats, rounded to 16 bits, as one 16-byte word
template <int DT>
__device__ __forceinline__ uint4 pack8(const float *v, float scale)
{
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h)
        o[h] = pack2<DT>(v[2 * h] * scale, v[2 * h + 1] * scale);  // one paired conversion
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------ row softmax, LPR lanes per row
// Rows of up to LPR * PER_LANE values live in registers: one read, one write.
// A warp serves 32 / LPR rows at a time (short rows do not leave lanes idle)
// and loads its next rows before reducing the current ones, so a load is in
// flight while the previous rows are reduced and written.
template <int DT, int PER_LANE, bool VEC, int LPR>
__global__ void __launch_bounds__(256, VEC ? 4 : 2) softmax_rows_warp_kernel(const uint16_t *__restrict__ X,
                                                                uint16_t *__restrict__ Y, int64_t rows, int cols)
{
    static_assert(LPR == 8 || LPR == 16 || LPR == 32, "lanes per row");
    constexpr int RPW = 32 / LPR;                   // rows per warp
    constexpr int NW = VEC ? PER_LANE / 8 : 1;      // 16-byte words a lane holds
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPR;                     // lane within its row
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t warp0 = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t group_stride = warps_total * RPW;

    uint4 w[NW];                                    // raw words (VEC)
    uint16_t e[VEC ? 1 : PER_LANE];                 // raw values (scalar path)
    auto load = [&](int64_t row) {
        if (row >= rows)
            return;
        const uint16_t *x = X + row * cols;
        if constexpr (VEC) {
#pragma unroll
            for (int s = 0; s < NW; ++s) {
                const int c = s * LPR * 8 + sub * 8;
                if (c < cols)
                    w[s] = __ldg(reinterpret_cast<const uint4 *>(x + c));
            }
        } else {
#pragma unroll
            for (int s = 0; s < PER_LANE; ++s) {
                const int c = s * LPR + sub;
                if (c < cols)
                    e[s] = __ldg(x + c);
            }
        }
    };
    int64_t row = warp0 * RPW + lane / LPR;
    load(row);
    // the loop runs while any row of the warp is live (shuffles need every lane)
    for (int64_t base = warp0 * RPW; base < rows; base += group_stride, row += group_stride) {
        const bool live = row < rows;
        float v[PER_LANE];
        if constexpr (VEC) {
#pragma unroll
            for (int s = 0; s < NW; ++s) {
                const int c = s * LPR * 8 + sub * 8;
                if (live && c < cols) {
                    unpack8<DT>(w[s], v + 8 * s);
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        v[8 * s + k] = -INFINITY;
                }
            }
        } else {
#pragma unroll
            for (int s = 0; s < PER_LANE; ++s)
                v[s] = (live && s * LPR + sub < cols) ? half_to_float<DT>(e[s]) : -INFINITY;
        }
        load(row + group_stride);  // next rows: in flight during this row's work
        float m = -INFINITY;
        static_assert(PER_LANE % 2 == 0, "pairs for the three-way max");
#pragma unroll
        for (int s = 0; s < PER_LANE; s += 2)
            m = fmax3(m, v[s], v[s + 1]);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float mb = live ? m * kLog2e : 0.0f;
        float sum = 0.0f;
#pragma unroll
        for (int s = 0; s < PER_LANE; ++s) {
            v[s] = exp2_approx_ftz(fmaf(v[s], kLog2e, -mb));  // -inf (padding) -> 0
            sum += v[s];
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (!live)
            continue;
        const float inv = 1.0f / sum;
        uint16_t *y = Y + row * cols;
        if constexpr (VEC) {
#pragma unroll
            for (int s = 0; s < NW; ++s) {
                const int c = s * LPR * 8 + sub * 8;
                if (c < cols)
                    *reinterpret_cast<uint4 *>(y + c) = pack8<DT>(v + 8 * s, inv);
            }
        } else {
#pragma unroll
            for (int s = 0; s < PER_LANE; ++s) {
                const int c = s * LPR + sub;
                if (c < cols)
                    y[c] = float_to_half<DT>(v[s] * inv);
            }
        }
    }
}

// ------------------------------------------------------------------ row softmax, one CTA per row, in registers
// Rows of up to THREADS * PER_THREAD values (16-byte aligned, a multiple of 8
// long) are read once into registers; block reductions through shared memory.
// The CTA's next row is loaded (as raw words) before the current one is
// reduced, so its loads are in flight during the reductions.
template <int DT, int PER_THREAD>
__global__ void __launch_bounds__(512, PER_THREAD <= 16 ? 3 : 2) softmax_rows_cta_regs_kernel(const uint16_t *__restrict__ X,
                                                                    uint16_t *__restrict__ Y, int64_t rows, int cols)
{
    constexpr int NW = PER_THREAD / 8;
    __shared__ float red[2][16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int step = blockDim.x * 8;
    uint4 w[NW];
    auto load = [&](int64_t row) {
        if (row >= rows)
            return;
        const uint16_t *x = X + row * cols;
#pragma unroll
        for (int s = 0; s < NW; ++s) {
            const int c = s * step + tid * 8;
            if (c < cols)
                w[s] = __ldg(reinterpret_cast<const uint4 *>(x + c));
        }
    };
    load(blockIdx.x);
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        float v[PER_THREAD];
#pragma unroll
        for (int s = 0; s < NW; ++s) {
            const int c = s * step + tid * 8;
            if (c < cols) {
                unpack8<DT>(w[s], v + 8 * s);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    v[8 * s + k] = -INFINITY;
            }
        }
        load(row + gridDim.x);
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < PER_THREAD; i += 2)
            m = fmax3(m, v[i], v[i + 1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        // red[0] holds maxima, red[1] sums: the barrier after the sums orders
        // this row's reads of red[0] before the next row's writes
        if (lane == 0)
            red[0][warp] = m;
        __syncthreads();
        m = red[0][0];
        for (int k = 1; k < nwarps; ++k)
            m = fmaxf(m, red[0][k]);
        const float mb = m * kLog2e;
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < PER_THREAD; ++i) {
            v[i] = exp2_approx_ftz(fmaf(v[i], kLog2e, -mb));
            sum += v[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0)
            red[1][warp] = sum;
        __syncthreads();
        sum = 0.0f;
        for (int k = 0; k < nwarps; ++k)
            sum += red[1][k];
        const float inv = 1.0f / sum;
        uint16_t *y = Y + row * cols;
#pragma unroll
        for (int s = 0; s < NW; ++s) {
            const int c = s * step + tid * 8;
            if (c < cols)
                *reinterpret_cast<uint4 *>(y + c) = pack8<DT>(v + 8 * s, inv);
        }
    }
}

// ------------------------------------------------------------------ row softmax, one CTA per row, in shared memory
// Rows too long for registers but short enough for shared memory (up to
// ~110,000 values).  One thread streams the row's 16-byte-aligned body into
// shared memory with bulk copies (the TMA engine, completion counted on an
// mbarrier); the few values before the first and after the last 16-byte
// boundary are loaded by plain loads.  The row sits in shared memory at the
// same offset from a 16-byte boundary as in global memory.  With two row
// buffers (rows up to ~55,000 values) the next row's copy runs while the
// current row is reduced and written, so HBM reads one row ahead.
// The wait for a copy is bounded; on expiry the kernel records
// ERR_ROW_COPY in the device error word and carries on (the row's output is
// then wrong, which tl_check_device reports), so no thread ever hangs.
constexpr unsigned ERR_ROW_COPY = 64u;

struct RowSplit {
    int mis;   // byte offset of the row start from a 16-byte boundary (even)
    int head;  // values before the first 16-byte boundary
    int nvec;  // 8-value words in the aligned body
};

__device__ __forceinline__ RowSplit split_row(const uint16_t *x, int cols)
{
    RowSplit r;
    r.mis = static_cast<int>(reinterpret_cast<uintptr_t>(x) & 15);
    r.head = min(((16 - r.mis) & 15) >> 1, cols);
    r.nvec = (cols - r.head) >> 3;
    return r;
}

template <int DT>
__global__ void __launch_bounds__(512) softmax_rows_smem_kernel(const uint16_t *__restrict__ X,
                                                                uint16_t *__restrict__ Y, int64_t rows, int cols,
                                                                int y_vec, int nbuf, int buf_bytes,
                                                                uint64_t timeout_ns)
{
    extern __shared__ __align__(128) uint8_t smem_dyn[];
    // row buffers from the first 128-byte boundary (the launch adds 128 bytes)
    uint8_t *srow_raw = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_dyn) + 127) &
                                                    ~static_cast<uintptr_t>(127));
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ float red_m[16], red_s[16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    if (tid == 0) {
        mbar_init(smem_addr(&bars[0]), 1);
        mbar_init(smem_addr(&bars[1]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    // one thread: start the copy of `row`'s body into buffer `buf`
    auto issue = [&](int64_t row, int buf) {
        const uint16_t *x = X + row * cols;
        const RowSplit sp = split_row(x, cols);
        const uint32_t bar = smem_addr(&bars[buf]);
        if (sp.nvec == 0) {
            mbar_arrive(bar);
            return;
        }
        const uint32_t bytes = static_cast<uint32_t>(sp.nvec) * 16u;
        const uint32_t dst = smem_addr(srow_raw + buf * buf_bytes + sp.mis + 2 * sp.head);
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x + sp.head);
        // checked build: the copy stays inside its row buffer, starts and ends on
        // 16-byte boundaries, and reads inside the row
        if (!check_ok(buf < nbuf && sp.mis + 2 * sp.head + static_cast<int>(bytes) <= buf_bytes && (dst & 15u) == 0 &&
                      (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && sp.head + 8 * sp.nvec <= cols)) {
            mbar_arrive(bar);  // complete the phase without the copy
            return;
        }
        fence_proxy_async_smem();  // earlier generic reads of this buffer come first
        mbar_arrive_expect_tx(bar, bytes);
        constexpr uint32_t CHUNK = 32768;
        for (uint32_t off = 0; off < bytes; off += CHUNK)
            bulk_load_g2s(dst + off, src + off, min(CHUNK, bytes - off), bar);
    };

    int it = 0;
    uint32_t phases = 0u;  // bit b: parity of buffer b's next phase
    if (tid == 0 && static_cast<int64_t>(blockIdx.x) < rows)
        issue(blockIdx.x, 0);
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x, ++it) {
        const int buf = nbuf == 2 ? (it & 1) : 0;
        const int64_t next = row + gridDim.x;
        if (nbuf == 2 && tid == 0 && next < rows)
            issue(next, buf ^ 1);  // its buffer was released by the barrier that ended the previous row
        const uint16_t *x = X + row * cols;
        uint16_t *y = Y + row * cols;
        const RowSplit sp = split_row(x, cols);
        uint16_t *sr = reinterpret_cast<uint16_t *>(srow_raw + buf * buf_bytes + sp.mis);
        const int body_end = sp.head + (sp.nvec << 3);
        for (int c = tid; c < sp.head; c += blockDim.x)
            sr[c] = x[c];
        for (int c = body_end + tid; c < cols; c += blockDim.x)
            sr[c] = x[c];
        {
            // bounded wait for the body (every thread)
            const uint32_t bar = smem_addr(&bars[buf]);
            const uint32_t parity = (phases >> buf) & 1u;
            if (!mbar_try_wait(bar, parity)) {
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar, parity)) {
                    if (global_timer_ns() - t0 > timeout_ns) {
                        atomicOr(&g_device_error, ERR_ROW_COPY);
                        break;
                    }
                }
            }
            phases ^= 1u << buf;
        }
        __syncthreads();  // head and tail visible to every thread

        // running (max, sum) in log2 units over the row in shared memory
        float m = -INFINITY, s = 0.0f;
        auto absorb = [&](float t) {
            if (t > m) {
                s = s * exp2_approx_ftz(m - t) + 1.0f;
                m = t;
            } else {
                s += exp2_approx_ftz(t - m);
            }
        };
        for (int c = tid; c < sp.head; c += blockDim.x)
            absorb(half_to_float<DT>(sr[c]) * kLog2e);
        const uint4 *body = reinterpret_cast<const uint4 *>(sr + sp.head);
        for (int i = tid; i < sp.nvec; i += blockDim.x) {
            float t[8];
            unpack8<DT>(body[i], t);
            float mx = t[0];
#pragma unroll
            for (int e = 1; e < 8; ++e)
                mx = fmaxf(mx, t[e]);
            mx *= kLog2e;
            if (mx > m) {
                s = (m == -INFINITY) ? 0.0f : s * exp2_approx_ftz(m - mx);
                m = mx;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e)
                s += exp2_approx_ftz(fmaf(t[e], kLog2e, -m));
        }
        for (int c = body_end + tid; c < cols; c += blockDim.x)
            absorb(half_to_float<DT>(sr[c]) * kLog2e);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
            const float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.0f : s * exp2_approx_ftz(m - mm)) + (m2 == -INFINITY ? 0.0f : s2 * exp2_approx_ftz(m2 - mm));
            m = mm;
        }
        if (lane == 0) {
            red_m[warp] = m;
            red_s[warp] = s;
        }
        __syncthreads();
        float M = -INFINITY;
        for (int k = 0; k < nwarps; ++k)
            M = fmaxf(M, red_m[k]);
        float S = 0.0f;
        for (int k = 0; k < nwarps; ++k)
            if (red_m[k] != -INFINITY)
                S += red_s[k] * exp2_approx_ftz(red_m[k] - M);
        const float inv = 1.0f / S;
        if (y_vec) {
            // y lies as far from a 16-byte boundary as x: whole words for the body
            for (int c = tid; c < sp.head; c += blockDim.x)
                y[c] = float_to_half<DT>(exp2_approx_ftz(fmaf(half_to_float<DT>(sr[c]), kLog2e, -M)) * inv);
            for (int i = tid; i < sp.nvec; i += blockDim.x) {
                float t[8];
                unpack8<DT>(body[i], t);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    t[e] = exp2_approx_ftz(fmaf(t[e], kLog2e, -M));
                __stcs(reinterpret_cast<uint4 *>(y + sp.head) + i, pack8<DT>(t, inv));
            }
            for (int c = body_end + tid; c < cols; c += blockDim.x)
                y[c] = float_to_half<DT>(exp2_approx_ftz(fmaf(half_to_float<DT>(sr[c]), kLog2e, -M)) * inv);
        } else {
            for (int c = tid; c < cols; c += blockDim.x)
                y[c] = float_to_half<DT>(exp2_approx_ftz(fmaf(half_to_float<DT>(sr[c]), kLog2e, -M)) * inv);
        }
        __syncthreads();  // the row buffer and red_* are free for the next row
        if (nbuf == 1 && tid == 0 && next < rows)
            issue(next, 0);
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
                s = s * exp2_approx_ftz(m - t) + 1.0f;
                m = t;
            } else {
                s += exp2_approx_ftz(t - m);
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
                s = (m == -INFINITY) ? 0.0f : s * exp2_approx_ftz(m - mx);
                m = mx;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e)
                s += exp2_approx_ftz(t[e] - m);
        }
        for (int64_t c = body_end + tid; c < cols; c += blockDim.x)
            absorb(half_to_float<DT>(x[c]) * kLog2e);
        // merge (m, s) across the warp, then across warps
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
            const float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.0f : s * exp2_approx_ftz(m - mm)) + (m2 == -INFINITY ? 0.0f : s2 * exp2_approx_ftz(m2 - mm));
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
                S += red_s[w] * exp2_approx_ftz(red_m[w] - M);
        __syncthreads();  // red_* reused by the next row
        const float inv = 1.0f / S;
        for (int64_t c = tid; c < head; c += blockDim.x)
            y[c] = float_to_half<DT>(exp2_approx_ftz(fmaf(half_to_float<DT>(x[c]), kLog2e, -M)) * inv);
        for (int64_t i = tid; i < nvec; i += blockDim.x) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + head) + i);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float a = exp2_approx_ftz(fmaf(half_to_float<DT>(static_cast<uint16_t>(ww[h] & 0xFFFFu)), kLog2e, -M)) * inv;
                const float b = exp2_approx_ftz(fmaf(half_to_float<DT>(static_cast<uint16_t>(ww[h] >> 16)), kLog2e, -M)) * inv;
                o[h] = float_to_half<DT>(a) | (static_cast<uint32_t>(float_to_half<DT>(b)) << 16);
            }
            reinterpret_cast<uint4 *>(y + head)[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        for (int64_t c = body_end + tid; c < cols; c += blockDim.x)
            y[c] = float_to_half<DT>(exp2_approx_ftz(fmaf(half_to_float<DT>(x[c]), kLog2e, -M)) * inv);
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
