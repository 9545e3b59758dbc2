// attention_kernel.cuh -- attention forward on sm_100a with an online softmax:
//
//     O = softmax(scale * Q K^T  [causal: key j > query i removed]) V
//     lse_i = log sum_j exp(scale * q_i . k_j)
//
// What it computes follows the TileLang GPU kernel design article, paragraph 6
// (query, key and value tiles; online softmax with a running maximum, a
// normaliser and rescaling; tiled tensor-core products; the full score matrix
// never written to global memory; causal and non-causal, checked against
// PyTorch's scaled dot-product attention, whose causal mask keeps j <= i).
//
// One CTA computes 128 query rows of one (batch, head).  For each block of 128
// keys:
//   S  = Q K^T          tcgen05.mma, fp32 in Tensor Memory (double-buffered)
//   P  = exp2(S' - m)   softmax warps, one query row per thread, written to
//                       shared memory in the 16-bit input type
//   Ot = P V            tcgen05.mma, fp32 in Tensor Memory (double-buffered)
//   O  = alpha O + Ot   the softmax warps' registers, one block behind, so the
//                       softmax of block j overlaps the P V product of j - 1
// Q and K tiles are K-major operands; V uses the same TMA boxes read as an
// N-major operand; P is K-major.  All in 128-byte swizzled layouts.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 2..3 idle, warps 4..11 softmax / output.  Warp w owns TMEM
// lanes 32*(w%4)..+31 (its query rows) and one half of each key block and of
// O's columns; the two warps of a lane quarter trade their row maxima and
// sums through shared memory under a 64-thread named barrier.
// Every wait is bounded; on expiry the kernel records it in the device error
// word, lets issued copies and MMAs land, frees TMEM and returns.
#pragma once

#include "gemm_kernel.cuh"

namespace tl {

struct AttnParams {
    int32_t Sq, Sk, BH;      // query and key lengths, batch * heads
    int32_t num_qtiles;
    int32_t causal;
    float scale_log2;        // softmax scale * log2(e)
    uint16_t *O;             // [BH][Sq][D]
    float *lse;              // [BH][Sq] natural log, or null
    uint64_t timeout_ns;
};

template <int D_>
struct AttnConfig {
    static constexpr int D = D_;
    static constexpr int BM = 128, BN = 128;
    static constexpr int KS = D == 128 ? 2 : 3;            // K / V ring depth
    static constexpr int ATOM_BYTES = 128 * 128;          // 128 rows x 64 16-bit values
    static constexpr int D_ATOMS = D / 64;
    static constexpr int Q_BYTES = D_ATOMS * ATOM_BYTES;
    static constexpr int KV_BYTES = D_ATOMS * ATOM_BYTES;  // one K (or V) block
    static constexpr int P_BYTES = 2 * ATOM_BYTES;        // 128 queries x 128 keys
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
    static constexpr int OFF_P = OFF_V + KS * KV_BYTES;
    static constexpr int OFF_X = OFF_P + 2 * P_BYTES;      // row max (then sum) exchange: [2 halves][128 rows]
    static constexpr int OFF_BAR = OFF_X + 2 * 128 * 4;
    // barrier map
    static constexpr int BAR_Q = 0, BAR_KF = 1, BAR_KE = 1 + KS, BAR_VF = 1 + 2 * KS, BAR_VE = 1 + 3 * KS;
    static constexpr int BAR_SF = 1 + 4 * KS, BAR_SE = BAR_SF + 2, BAR_PF = BAR_SE + 2, BAR_PE = BAR_PF + 2;
    static constexpr int BAR_OF = BAR_PE + 2, BAR_OE = BAR_OF + 2, BAR_DRAIN = BAR_OE + 2;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static constexpr int SMEM_USED = OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;
    static constexpr int THREADS = 384;
    // registers a thread: warpgroup 0 (producer, MMA, two idle warps) gives
    // up registers to the two softmax warpgroups; the launch must provide
    // at least LAUNCH_REGS a thread for the split to fit
    static constexpr int REGS_CONTROL = 80, REGS_SOFTMAX = 208;
    static constexpr int LAUNCH_REGS = (128 * REGS_CONTROL + 256 * REGS_SOFTMAX + THREADS - 1) / THREADS;
    static constexpr int FIRST_SOFTMAX_WARP = 4;
    static constexpr int TMEM_S = 0, TMEM_O = 256;  // S buffers at columns 0 / 128, O at 256 / 256 + D
    static constexpr int SOFTMAX_WARPS = 8;  // two per TMEM lane quarter: halves of the keys and of O
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class CF, int DT>
__global__ void __launch_bounds__(384, 1)
    attention_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const AttnParams p)
{
    constexpr int D = CF::D;
    constexpr int KS = CF::KS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // heaviest tiles first when causal (later query tiles see more keys)
    const int qt = p.causal ? p.num_qtiles - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
    const int bh = static_cast<int>(blockIdx.y);
    const int q0 = qt * CF::BM;
    const int kblocks_all = (p.Sk + CF::BN - 1) / CF::BN;
    const int nb = p.causal ? min(kblocks_all, (q0 + CF::BM - 1) / CF::BN + 1) : kblocks_all;

    const uint32_t sQ = smem_addr(smem + CF::OFF_Q);
    const uint32_t sK = smem_addr(smem + CF::OFF_K);
    const uint32_t sV = smem_addr(smem + CF::OFF_V);
    uint8_t *pbuf = smem + CF::OFF_P;
    const uint32_t sP = smem_addr(pbuf);
    const uint32_t bar0 = smem_addr(smem + CF::OFF_BAR);
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CF::OFF_BAR + CF::NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    if (threadIdx.x == 0) {
        mbar_init(bar(CF::BAR_Q), 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(bar(CF::BAR_KF + s), 1);
            mbar_init(bar(CF::BAR_KE + s), 1);
            mbar_init(bar(CF::BAR_VF + s), 1);
            mbar_init(bar(CF::BAR_VE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(CF::BAR_SF + b), 1);
            mbar_init(bar(CF::BAR_SE + b), CF::SOFTMAX_WARPS);
            mbar_init(bar(CF::BAR_PF + b), CF::SOFTMAX_WARPS);
            mbar_init(bar(CF::BAR_PE + b), 1);
            mbar_init(bar(CF::BAR_OF + b), 1);
            mbar_init(bar(CF::BAR_OE + b), CF::SOFTMAX_WARPS);
        }
        mbar_init(bar(CF::BAR_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmap_q);
        tma_prefetch_map(&tmap_k);
        tma_prefetch_map(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t timeout = p.timeout_ns;
    grid_dependency_wait();
    grid_launch_dependents();

    // issued copies per ring slot (bit) and the phase parity of the last fill
    uint32_t q_issued = 0, k_issued = 0, k_par = 0, v_issued = 0, v_par = 0;
    // The register split is taken at the top of each warpgroup's branch, so
    // the compiler allocates each branch under its own budget.
    if (warp < CF::FIRST_SOFTMAX_WARP) {
        regs_decrease<CF::REGS_CONTROL>();
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                bool ok = true;
                mbar_arrive_expect_tx(bar(CF::BAR_Q), CF::Q_BYTES);
    #pragma unroll
                for (int a = 0; a < CF::D_ATOMS; ++a)
                    tma_load_3d(sQ + a * CF::ATOM_BYTES, &tmap_q, bar(CF::BAR_Q), 64 * a, q0, bh);
                q_issued = 1;
                int st = 0;
                uint32_t ph = 0;
                for (int j = 0; ok && j < nb; ++j) {
                    if (!wait_bounded(bar(CF::BAR_KE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(CF::BAR_KF + st), CF::KV_BYTES);
    #pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d(sK + st * CF::KV_BYTES + a * CF::ATOM_BYTES, &tmap_k, bar(CF::BAR_KF + st), 64 * a,
                                    j * CF::BN, bh);
                    k_issued |= 1u << st;
                    k_par = (k_par & ~(1u << st)) | (ph << st);
                    if (!wait_bounded(bar(CF::BAR_VE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(CF::BAR_VF + st), CF::KV_BYTES);
    #pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d(sV + st * CF::KV_BYTES + a * CF::ATOM_BYTES, &tmap_v, bar(CF::BAR_VF + st), 64 * a,
                                    j * CF::BN, bh);
                    v_issued |= 1u << st;
                    v_par = (v_par & ~(1u << st)) | (ph << st);
                    if (++st == KS) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t IDESC_QK = mma_idesc_f16(DT, 128, 128, 0, 0);  // both K-major
                constexpr uint32_t IDESC_PV = mma_idesc_f16(DT, 128, D, 0, 1);    // P K-major, V N-major
                const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
                const uint64_t k_desc0 = smem_desc_sw128(sK, 16, 1024);
                const uint64_t p_desc0 = smem_desc_sw128(sP, 16, 1024);
                const uint64_t v_desc0 = smem_desc_sw128(sV, CF::ATOM_BYTES, 1024);
                // K-major operand, K step k of 16: atom k / 4 (+16 KB), +32 B inside it
                auto kmaj = [](int k) { return static_cast<uint64_t>(((k >> 2) * CF::ATOM_BYTES + (k & 3) * 32) >> 4); };
                bool ok = wait_bounded(bar(CF::BAR_Q), 0, abort_flag, timeout, ERR_MMA_DATA);
                tc_fence_after_sync();
                int kst = 0, vst = 0;
                uint32_t kph = 0, vph = 0;
                auto pv = [&](int i) -> bool {
                    const int b = i & 1;
                    const uint32_t bp = static_cast<uint32_t>(i >> 1) & 1u;
                    if (!wait_bounded(bar(CF::BAR_PF + b), bp, abort_flag, timeout, ERR_MMA_DATA))
                        return false;
                    if (!wait_bounded(bar(CF::BAR_VF + vst), vph, abort_flag, timeout, ERR_MMA_DATA))
                        return false;
                    if (!wait_bounded(bar(CF::BAR_OE + b), bp ^ 1u, abort_flag, timeout, ERR_MMA_ACC))
                        return false;
                    tc_fence_after_sync();
                    const uint32_t d_o = tmem_base + static_cast<uint32_t>(CF::TMEM_O + b * D);
                    const uint64_t pd = p_desc0 + ((b * CF::P_BYTES) >> 4);
                    const uint64_t vd = v_desc0 + ((vst * CF::KV_BYTES) >> 4);
    #pragma unroll
                    for (int k = 0; k < CF::BN / 16; ++k)  // 16 keys per step: +2048 B down V's rows
                        tc_mma_f16(d_o, pd + kmaj(k), vd + ((2048 * k) >> 4), IDESC_PV, k != 0 ? 1u : 0u);
                    tc_commit(bar(CF::BAR_OF + b));
                    tc_commit(bar(CF::BAR_VE + vst));
                    tc_commit(bar(CF::BAR_PE + b));
                    if (++vst == KS) {
                        vst = 0;
                        vph ^= 1u;
                    }
                    return true;
                };
                for (int j = 0; ok && j < nb; ++j) {
                    const int b = j & 1;
                    const uint32_t bp = static_cast<uint32_t>(j >> 1) & 1u;
                    if (!wait_bounded(bar(CF::BAR_KF + kst), kph, abort_flag, timeout, ERR_MMA_DATA) ||
                        !wait_bounded(bar(CF::BAR_SE + b), bp ^ 1u, abort_flag, timeout, ERR_MMA_ACC)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_s = tmem_base + static_cast<uint32_t>(CF::TMEM_S + b * 128);
                    const uint64_t kd = k_desc0 + ((kst * CF::KV_BYTES) >> 4);
    #pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_mma_f16(d_s, q_desc + kmaj(k), kd + kmaj(k), IDESC_QK, k != 0 ? 1u : 0u);
                    tc_commit(bar(CF::BAR_SF + b));
                    tc_commit(bar(CF::BAR_KE + kst));
                    if (++kst == KS) {
                        kst = 0;
                        kph ^= 1u;
                    }
                    if (j >= 1 && !pv(j - 1))
                        ok = false;
                }
                if (ok && nb >= 1)
                    pv(nb - 1);
                tc_commit(bar(CF::BAR_DRAIN));
                wait_drain(bar(CF::BAR_DRAIN), 0, timeout);
            }
            __syncwarp();
        }
    } else {
        regs_increase<CF::REGS_SOFTMAX>();
        // ------------------------------------------------------------ softmax and output
        const int q = warp & 3;
        const int half = (warp - CF::FIRST_SOFTMAX_WARP) >> 2;  // keys [64 half, +64) of a block; O columns [D/2 half, +D/2)
        const int r = q * 32 + lane;       // row of the tile (TMEM lane)
        const int row = q0 + r;            // query index
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        constexpr int DH = D / 2;
        // The two warps of a lane quarter trade one float per row through
        // xbuf[half][r] between two 64-thread named barriers.  Both warps run
        // every iteration and every barrier even after an error (the work is
        // skipped, the barriers are not), so neither can be left waiting.
        float *xbuf = reinterpret_cast<float *>(smem + CF::OFF_X);
        const uint32_t pair_bar = 1 + q;
        auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory"); };
        auto exchange = [&](float v) -> float {
            xbuf[half * 128 + r] = v;
            pair_sync();
            const float other = xbuf[(half ^ 1) * 128 + r];
            pair_sync();  // both read before either writes again
            return other;
        };
        // bounded wait whose outcome is the same for the whole warp
        auto wait_warp = [&](int id, uint32_t parity) -> bool {
            const bool w = wait_bounded(bar(id), parity, abort_flag, timeout, ERR_EPILOGUE);
            return __all_sync(0xffffffffu, w);
        };
        float o[DH];
#pragma unroll
        for (int i = 0; i < DH; ++i)
            o[i] = 0.0f;
        // m: running row maximum (log2 units), shared by both halves; l: this
        // half's running sum of weights against m
        float m = -INFINITY, l = 0.0f, alpha_prev = 0.0f;
        bool ok = true;

        // fold this warp's half of O_tmp of block i (against the max of block i) into o
        auto fold = [&](int i, float alpha) -> bool {
            const int b = i & 1;
            const uint32_t bp = static_cast<uint32_t>(i >> 1) & 1u;
            if (!wait_warp(CF::BAR_OF + b, bp))
                return false;
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t t[32];
                tmem_load_32cols(tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_O + b * D + half * DH + 32 * c), t);
                tmem_load_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    o[32 * c + e] = fmaf(o[32 * c + e], alpha, __uint_as_float(t[e]));
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(CF::BAR_OE + b));
            return true;
        };

        for (int j = 0; j < nb; ++j) {
            const int b = j & 1;
            const uint32_t bp = static_cast<uint32_t>(j >> 1) & 1u;
            // this warp's 64 scores of the row, held in registers
            uint32_t sv[64];
            if (ok)
                ok = wait_warp(CF::BAR_SF + b, bp);
            if (ok) {
                tc_fence_after_sync();
                const uint32_t s_addr = tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_S + b * 128 + half * 64);
                tmem_load_32cols(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_load_32cols(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_load_wait();
                // S read: the buffer goes back to the MMA warp
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(CF::BAR_SE + b));
            }
            const int key0 = j * CF::BN + half * 64;
            int key_end = min(p.Sk, key0 + 64);
            if (p.causal)
                key_end = min(key_end, row + 1);
            const int nvalid = ok ? key_end - key0 : 0;  // <= 0: none of this half is visible to the row
            // blocks wholly inside every row's range (all but the ragged last
            // block and the causal diagonal) skip the per-key masks
            const bool whole = __all_sync(0xffffffffu, nvalid >= 64);
            if (!whole) {
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (e >= nvalid)
                        sv[e] = __float_as_uint(-INFINITY);
            }
            // row maximum of the raw scores; scaling after the max is exact
            // (rounding of x * scale is monotone and scale > 0)
            float mx;
            {
                float t[8];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float *f = reinterpret_cast<const float *>(&sv[8 * g]);
                    t[g] = fmax3(fmax3(f[0], f[1], f[2]), fmax3(f[3], f[4], f[5]), fmaxf(f[6], f[7]));
                }
                mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]), fmaxf(t[6], t[7]));
            }
            mx *= p.scale_log2;
            const float m_new = fmaxf(m, fmaxf(mx, exchange(mx)));
            const float m_ref = m_new == -INFINITY ? 0.0f : m_new;  // no valid key yet: all weights 0
            const float alpha = exp2_approx_ftz(m - m_ref);        // 0 when m is -inf
            if (!ok)
                continue;
            // weights, their sum, and this half of P (16-bit) into shared memory
            if (j >= 2 && !(ok = wait_warp(CF::BAR_PE + b, bp ^ 1u)))
                continue;
            uint8_t *prow = pbuf + b * CF::P_BYTES + half * CF::ATOM_BYTES + r * 128;
            float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums: shorter add chains
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t pk[4];
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const int e = 8 * i + 2 * e2;
                    // masked scores are -inf: 2^-inf = 0
                    const float w0 = exp2_approx_ftz(fmaf(__uint_as_float(sv[e]), p.scale_log2, -m_ref));
                    const float w1 = exp2_approx_ftz(fmaf(__uint_as_float(sv[e + 1]), p.scale_log2, -m_ref));
                    part[e2] += w0 + w1;
                    pk[e2] = pack2<DT>(w0, w1);
                }
                // keys 8i .. 8i+7 of this half: 16-byte chunk i, swizzled by row
                *reinterpret_cast<uint4 *>(prow + ((i ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            const float sum = (part[0] + part[1]) + (part[2] + part[3]);
            // P written: visible to the tensor core
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(CF::BAR_PF + b));
            l = l * alpha + sum;
            m = m_new;
            if (j >= 1)
                ok = fold(j - 1, alpha_prev);
            alpha_prev = alpha;
        }
        if (ok && nb >= 1)
            ok = fold(nb - 1, alpha_prev);
        l += exchange(l);  // a + b == b + a: both halves get the same total

        if (ok && row < p.Sq) {
            const float inv = 1.0f / l;
            uint16_t *orow = p.O + (static_cast<size_t>(bh) * p.Sq + row) * D + half * DH;
#pragma unroll
            for (int c = 0; c < DH / 8; ++c) {
                uint4 w;
                w.x = pack2<DT>(o[8 * c] * inv, o[8 * c + 1] * inv);
                w.y = pack2<DT>(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                w.z = pack2<DT>(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                w.w = pack2<DT>(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                reinterpret_cast<uint4 *>(orow)[c] = w;
            }
            if (p.lse && half == 0)
                p.lse[static_cast<size_t>(bh) * p.Sq + row] = m * 0.69314718055994531f + logf(l);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        if (q_issued)
            wait_drain(bar(CF::BAR_Q), 0, timeout);
        for (int s = 0; s < KS; ++s) {
            if (k_issued & (1u << s))
                wait_drain(bar(CF::BAR_KF + s), (k_par >> s) & 1u, timeout);
            if (v_issued & (1u << s))
                wait_drain(bar(CF::BAR_VF + s), (v_par >> s) & 1u, timeout);
        }
    }
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1)
        tmem_dealloc(tmem_base, 512);
}

} // namespace tl
