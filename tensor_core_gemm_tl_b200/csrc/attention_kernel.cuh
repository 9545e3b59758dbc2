// attention_kernel.cuh -- attention forward on sm_100a, two query tiles per CTA
// in ping-pong:
//
//     O = softmax(scale * Q K^T  [causal: key j > query i removed]) V
//     lse_i = log sum_j exp(scale * q_i . k_j)
//
// What it computes follows the TileLang GPU kernel design article, paragraph 6
// (query, key and value tiles; online softmax with a running maximum, a
// normaliser and rescaling; the score matrix never written to global memory;
// causal and non-causal, checked against PyTorch's scaled dot-product
// attention, whose causal mask keeps j <= i).
//
// One CTA computes two 128-row query tiles (Q0, Q1) of one (batch, head)
// against the same stream of 128-key blocks of K and V.  Tensor Memory (512
// columns) holds, per tile i, S_i (128 fp32 columns) and the output
// accumulator O_i (D fp32 columns).  For each key block j:
//
//   S_i = Q_i K_j^T       tcgen05.mma (A, B from shared memory) into S_i
//   P_i = 2^(S_i' - m_i)  the tile's softmax warpgroup, one query row per
//                         thread: 16-bit weights written with tcgen05.st over
//                         S_i's first 64 columns (head_dim 128) or into
//                         columns of their own (head_dim 64)
//   O_i += P_i V_j        tcgen05.mma with A = P_i read from Tensor Memory
//
// With head_dim 128 the MMA thread issues PV_0(j), S_0(j+1), PV_1(j),
// S_1(j+1), ...: while one warpgroup turns S into P, the tensor core works on
// the other tile; S_i(j+1) overwrites the columns PV_i(j) reads, so it is
// issued only once PV_i(j) has completed.  With head_dim 64 it issues
// S_0(j+1), S_1(j+1) as soon as the softmax has read S_i(j), then PV_0(j),
// PV_1(j); the softmax writes P_i(j+1) once PV_i(j) has completed.  The running maximum m_i used for P only moves when a row's new
// maximum exceeds it by more than 2^8: then (rarely, after the first blocks)
// the warp multiplies its rows of O_i by 2^(m_old - m_new) in Tensor Memory
// before P_i(j) is released; otherwise the weights stay below 256.
//
// Warp roles (384 threads): warp 0 TMA producer (Q0, Q1 once; K and V blocks
// through rings), warp 1 TMEM allocator and MMA issuer, warps 2..3 idle,
// warps 4..7 softmax of tile 0, warps 8..11 softmax of tile 1 (warp w owns
// TMEM lanes 32*(w%4)..+31).  Every wait is bounded; on expiry the kernel
// records it in the device error word, lets issued copies and MMAs land,
// frees TMEM and returns.
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
    static constexpr int BM = 128, BN = 128, TILES = 2;
    static constexpr int KS = D == 128 ? 2 : 4;             // K and V ring depth
    static constexpr int ATOM_BYTES = 128 * 128;           // 128 rows x 64 16-bit values
    static constexpr int D_ATOMS = D / 64;
    static constexpr int Q_BYTES = D_ATOMS * ATOM_BYTES;   // one query tile
    static constexpr int KV_BYTES = D_ATOMS * ATOM_BYTES;  // one K (or V) block
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILES * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + KS * KV_BYTES;
    // barrier map
    static constexpr int BAR_Q = 0, BAR_KF = 1, BAR_KE = 1 + KS, BAR_VF = 1 + 2 * KS, BAR_VE = 1 + 3 * KS;
    static constexpr int BAR_SF = 1 + 4 * KS;   // [tile]: S_i(j) in Tensor Memory
    static constexpr int BAR_PF = BAR_SF + 2;   // [tile]: P_i(j) in Tensor Memory (4 warps arrive)
    static constexpr int BAR_PV = BAR_PF + 2;   // [tile]: O_i += P_i(j) V_j completed
    static constexpr int BAR_SE = BAR_PV + 2;   // [tile]: S_i(j) read into registers (4 warps; separate P only)
    static constexpr int BAR_DRAIN = BAR_SE + 2;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static constexpr int SMEM_USED = OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;
    static constexpr int THREADS = 384;
    static constexpr int FIRST_SOFTMAX_WARP = 4;
    static constexpr int REGS_CONTROL = 64, REGS_SOFTMAX = 216;
    static constexpr int LAUNCH_REGS = (128 * REGS_CONTROL + 256 * REGS_SOFTMAX + THREADS - 1) / THREADS;
    static constexpr int TMEM_S = 0, TMEM_O = 256;  // S_i at 128 i, O_i at 256 + D i
    // With D = 64 Tensor Memory has room for P_i in columns of its own (at
    // 384 + 64 i): S_i(j+1) can then be computed as soon as the softmax has
    // read S_i(j), while P_i(j) waits for its P V.  With D = 128, P_i(j) is
    // written over the first 64 columns of S_i.
    static constexpr bool SEPARATE_P = D == 64;
    static constexpr int TMEM_P = 256 + 2 * D;
    __host__ __device__ static constexpr int p_col(int i) { return SEPARATE_P ? TMEM_P + 64 * i : TMEM_S + 128 * i; }
    static_assert(!SEPARATE_P || TMEM_P + 128 <= 512, "Tensor Memory columns");
    static constexpr float RESCALE_LOG2 = 8.0f;     // m moves when a row maximum exceeds it by 2^8
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

    // CTA pairs of query tiles.  Non-causal: pairs along x, so the CTAs that
    // start together share a head's K and V in L2.  Causal: heads along x and
    // the pairs reversed along y, so every head's heaviest pair starts first.
    const int num_pairs = (p.num_qtiles + 1) / 2;
    const int pair_idx = static_cast<int>(p.causal ? blockIdx.y : blockIdx.x);
    const int qp = p.causal ? num_pairs - 1 - pair_idx : pair_idx;
    const int bh = static_cast<int>(p.causal ? blockIdx.x : blockIdx.y);
    const int q0 = qp * 2 * CF::BM;  // first query row of tile 0
    const int kblocks_all = (p.Sk + CF::BN - 1) / CF::BN;
    // key blocks each tile visits (a tile past the end of the queries visits none)
    auto blocks_of = [&](int t0) {
        return t0 >= p.Sq ? 0 : p.causal ? min(kblocks_all, (t0 + CF::BM - 1) / CF::BN + 1) : kblocks_all;
    };
    const int nb0 = blocks_of(q0), nb1 = blocks_of(q0 + CF::BM);
    auto nbt = [&](int i) { return i ? nb1 : nb0; };
    const int nbmax = max(nb0, nb1);

    const uint32_t sQ = smem_addr(smem + CF::OFF_Q);
    const uint32_t sK = smem_addr(smem + CF::OFF_K);
    const uint32_t sV = smem_addr(smem + CF::OFF_V);
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(CF::BAR_SF + i), 1);
            mbar_init(bar(CF::BAR_PF + i), 4);
            mbar_init(bar(CF::BAR_PV + i), 1);
            mbar_init(bar(CF::BAR_SE + i), 4);
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
    if (warp < CF::FIRST_SOFTMAX_WARP) {
        regs_decrease<CF::REGS_CONTROL>();
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                bool ok = true;
                mbar_arrive_expect_tx(bar(CF::BAR_Q), 2 * CF::Q_BYTES);
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d(sQ + i * CF::Q_BYTES + a * CF::ATOM_BYTES, &tmap_q, bar(CF::BAR_Q), 64 * a,
                                    q0 + i * CF::BM, bh);
                q_issued = 1;
                int st = 0;
                uint32_t ph = 0;
                for (int j = 0; ok && j < nbmax; ++j) {
                    if (!wait_bounded(bar(CF::BAR_KE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(CF::BAR_KF + st), CF::KV_BYTES);
#pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d(sK + st * CF::KV_BYTES + a * CF::ATOM_BYTES, &tmap_k, bar(CF::BAR_KF + st),
                                    64 * a, j * CF::BN, bh);
                    k_issued |= 1u << st;
                    k_par = (k_par & ~(1u << st)) | (ph << st);
                    if (!wait_bounded(bar(CF::BAR_VE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(CF::BAR_VF + st), CF::KV_BYTES);
#pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d(sV + st * CF::KV_BYTES + a * CF::ATOM_BYTES, &tmap_v, bar(CF::BAR_VF + st),
                                    64 * a, j * CF::BN, bh);
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
                constexpr uint32_t IDESC_QK = mma_idesc_f16(DT, 128, 128, 0, 0);  // Q, K both K-major
                constexpr uint32_t IDESC_PV = mma_idesc_f16(DT, 128, D, 0, 1);    // P K-major (TMEM), V N-major
                const uint64_t k_desc0 = smem_desc_sw128(sK, 16, 1024);
                const uint64_t v_desc0 = smem_desc_sw128(sV, CF::ATOM_BYTES, 1024);
                // K-major operand, K step k of 16: atom k / 4 (+16 KB), +32 B inside it
                auto kmaj = [](int k) { return static_cast<uint64_t>(((k >> 2) * CF::ATOM_BYTES + (k & 3) * 32) >> 4); };
                int kst = 0, vst = 0;
                uint32_t kph = 0, vph = 0;
                bool ok = wait_bounded(bar(CF::BAR_Q), 0, abort_flag, timeout, ERR_MMA_DATA);
                auto issue_s = [&](int i) {  // S_i = Q_i K^T from the current K slot
                    const uint64_t q_desc = smem_desc_sw128(sQ + i * CF::Q_BYTES, 16, 1024);
                    const uint64_t kd = k_desc0 + ((kst * CF::KV_BYTES) >> 4);
                    const uint32_t d_s = tmem_base + static_cast<uint32_t>(CF::TMEM_S + i * 128);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_mma_f16(d_s, q_desc + kmaj(k), kd + kmaj(k), IDESC_QK, k != 0 ? 1u : 0u);
                    tc_commit(bar(CF::BAR_SF + i));
                };
                auto issue_pv = [&](int i, int j) {  // O_i (+)= P_i V from the current V slot
                    const uint32_t d_o = tmem_base + static_cast<uint32_t>(CF::TMEM_O + i * D);
                    const uint32_t a_p = tmem_base + static_cast<uint32_t>(CF::p_col(i));
                    const uint64_t vd = v_desc0 + ((vst * CF::KV_BYTES) >> 4);
#pragma unroll
                    for (int k = 0; k < CF::BN / 16; ++k)  // 16 keys: 8 columns of P, 2048 B down V
                        tc_mma_f16_ts(d_o, a_p + 8 * k, vd + ((2048 * k) >> 4), IDESC_PV,
                                      (j > 0 || k > 0) ? 1u : 0u);
                    tc_commit(bar(CF::BAR_PV + i));
                };
                // prologue: S_0(0), S_1(0)
                if (ok && nbmax > 0) {
                    ok = wait_bounded(bar(CF::BAR_KF + kst), kph, abort_flag, timeout, ERR_MMA_DATA);
                    if (ok) {
                        tc_fence_after_sync();
                        for (int i = 0; i < 2; ++i)
                            if (nbt(i) > 0)
                                issue_s(i);
                        tc_commit(bar(CF::BAR_KE + kst));
                        if (++kst == KS) {
                            kst = 0;
                            kph ^= 1u;
                        }
                    }
                }
                for (int j = 0; ok && j < nbmax; ++j) {
                    const uint32_t jp = static_cast<uint32_t>(j) & 1u;
                    bool k_ready = false;  // K(j + 1) waited for
                    if constexpr (CF::SEPARATE_P) {
                        // S_i(j + 1) as soon as the softmax holds S_i(j) in registers
                        for (int i = 0; ok && i < 2; ++i) {
                            if (j + 1 < nbt(i)) {
                                if ((!k_ready && !wait_bounded(bar(CF::BAR_KF + kst), kph, abort_flag, timeout,
                                                               ERR_MMA_DATA)) ||
                                    !wait_bounded(bar(CF::BAR_SE + i), jp, abort_flag, timeout, ERR_MMA_ACC)) {
                                    ok = false;
                                    break;
                                }
                                k_ready = true;
                                tc_fence_after_sync();
                                issue_s(i);
                            }
                        }
                        if (!ok)
                            break;
                        if (!wait_bounded(bar(CF::BAR_VF + vst), vph, abort_flag, timeout, ERR_MMA_DATA)) {
                            ok = false;
                            break;
                        }
                        for (int i = 0; ok && i < 2; ++i) {
                            if (j < nbt(i)) {
                                if (!wait_bounded(bar(CF::BAR_PF + i), jp, abort_flag, timeout, ERR_MMA_DATA)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after_sync();
                                issue_pv(i, j);
                            }
                        }
                        if (!ok)
                            break;
                        tc_commit(bar(CF::BAR_VE + vst));  // V(j) free once the P V of block j are done
                    } else {
                        if (!wait_bounded(bar(CF::BAR_VF + vst), vph, abort_flag, timeout, ERR_MMA_DATA)) {
                            ok = false;
                            break;
                        }
                        for (int i = 0; ok && i < 2; ++i) {
                            if (j < nbt(i)) {
                                if (!wait_bounded(bar(CF::BAR_PF + i), jp, abort_flag, timeout, ERR_MMA_DATA)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after_sync();
                                issue_pv(i, j);
                            }
                            if (i == 1)
                                tc_commit(bar(CF::BAR_VE + vst));  // V(j) free once the last P V of block j is done
                            if (j + 1 < nbt(i)) {
                                // S_i(j + 1) overwrites the P_i(j) that PV_i(j) reads: wait for it
                                if ((!k_ready && !wait_bounded(bar(CF::BAR_KF + kst), kph, abort_flag, timeout,
                                                               ERR_MMA_DATA)) ||
                                    !wait_bounded(bar(CF::BAR_PV + i), jp, abort_flag, timeout, ERR_MMA_ACC)) {
                                    ok = false;
                                    break;
                                }
                                k_ready = true;
                                tc_fence_after_sync();
                                issue_s(i);
                            }
                        }
                        if (!ok)
                            break;
                    }
                    if (++vst == KS) {
                        vst = 0;
                        vph ^= 1u;
                    }
                    if (k_ready) {
                        tc_commit(bar(CF::BAR_KE + kst));
                        if (++kst == KS) {
                            kst = 0;
                            kph ^= 1u;
                        }
                    }
                }
                tc_commit(bar(CF::BAR_DRAIN));
                wait_drain(bar(CF::BAR_DRAIN), 0, timeout);
            }
            __syncwarp();
        }
    } else {
        regs_increase<CF::REGS_SOFTMAX>();
        // ------------------------------------------------------------ softmax and output of one tile
        const int tile = (warp - CF::FIRST_SOFTMAX_WARP) >> 2;
        const int q = warp & 3;
        const int r = q * 32 + lane;                  // row of the tile (TMEM lane)
        const int row = q0 + tile * CF::BM + r;       // query index
        const int nb = nbt(tile);
        // checked build: this tile's Tensor Memory columns (S, P, O) inside the
        // 512 allocated, its key blocks inside K
        check_ok(CF::TMEM_S + tile * 128 + 128 <= 512 && CF::p_col(tile) + 64 <= 512 &&
                 CF::TMEM_O + tile * D + D <= 512 && nb <= kblocks_all && bh < p.BH);
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t s_addr = tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_S + tile * 128);
        const uint32_t p_addr =
            CF::SEPARATE_P ? tmem_base + lane_base + static_cast<uint32_t>(CF::p_col(tile)) : s_addr;
        const uint32_t o_addr = tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_O + tile * D);
        auto wait_warp = [&](int id, uint32_t parity) -> bool {
            const bool w = wait_bounded(bar(id), parity, abort_flag, timeout, ERR_EPILOGUE);
            return __all_sync(0xffffffffu, w);
        };
        // m: the reference maximum of the row's weights (log2 units); l: sum of
        // the weights against m
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; ok && j < nb; ++j) {
            const uint32_t jp = static_cast<uint32_t>(j) & 1u;
            if (!(ok = wait_warp(CF::BAR_SF + tile, jp)))
                break;
            tc_fence_after_sync();
            // S in two waves of 64 columns: the maximum of the first runs while
            // the second is still arriving
            uint32_t sv[128];
            tmem_load_32cols(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_load_32cols(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_load_wait();
            tmem_load_32cols(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
            tmem_load_32cols(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
            float t[16];  // maxima of groups of 8 raw scores
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float *f = reinterpret_cast<const float *>(&sv[8 * g]);
                t[g] = fmax3(fmax3(f[0], f[1], f[2]), fmax3(f[3], f[4], f[5]), fmaxf(f[6], f[7]));
            }
            tmem_load_wait();
            if constexpr (CF::SEPARATE_P) {
                // S_i(j) is in registers: its columns may take S_i(j + 1)
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(CF::BAR_SE + tile));
            }
            const int key0 = j * CF::BN;
            int nvalid = min(p.Sk, key0 + CF::BN) - key0;
            if (p.causal)
                nvalid = min(nvalid, row + 1 - key0);
            if (!__all_sync(0xffffffffu, nvalid >= CF::BN)) {
                // masked keys count neither in the maximum nor in the weights
#pragma unroll
                for (int e = 0; e < 128; ++e)
                    if (e >= nvalid)
                        sv[e] = __float_as_uint(-INFINITY);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float *f = reinterpret_cast<const float *>(&sv[8 * g]);
                    t[g] = fmax3(fmax3(f[0], f[1], f[2]), fmax3(f[3], f[4], f[5]), fmaxf(f[6], f[7]));
                }
            }
            float mx;
            {
#pragma unroll
                for (int g = 8; g < 16; ++g) {
                    const float *f = reinterpret_cast<const float *>(&sv[8 * g]);
                    t[g] = fmax3(fmax3(f[0], f[1], f[2]), fmax3(f[3], f[4], f[5]), fmaxf(f[6], f[7]));
                }
#pragma unroll
                for (int g = 0; g < 8; ++g)
                    t[g] = fmaxf(t[g], t[g + 8]);
                mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[4], t[5]), fmaxf(t[6], t[7]));
            }
            mx *= p.scale_log2;
            // move the reference maximum only when the weights would exceed 2^8
            const bool resc = mx > m + CF::RESCALE_LOG2;
            const float m_new = resc ? mx : m;
            const float m_ref = m_new == -INFINITY ? 0.0f : m_new;  // no visible key yet: all weights 0
            const float alpha = resc ? exp2_approx_ftz(m - m_ref) : 1.0f;  // 0 when m is -inf
            if constexpr (CF::SEPARATE_P) {
                // P_i's columns are free once PV_i(j - 1) has read them
                if (j > 0 && !(ok = wait_warp(CF::BAR_PV + tile, jp ^ 1u)))
                    break;
                tc_fence_after_sync();
            }
            // keys in pairs: the exponent argument and the running sums two
            // lanes per instruction
            const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 negm2 = make_float2(-m_ref, -m_ref);
            float2 part[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                              make_float2(0.0f, 0.0f)};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int e2 = 0; e2 < 32; ++e2) {
                    const int e = 64 * h + 2 * e2;
                    const float2 x = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), scale2, negm2);
                    const float2 w = make_float2(exp2_approx_ftz(x.x), exp2_approx_ftz(x.y));
                    part[e2 & 3] = fadd2(part[e2 & 3], w);
                    pk[e2] = pack2<DT>(w.x, w.y);  // keys 2 e2, 2 e2 + 1 of this half: one 32-bit column
                }
                tmem_store_32cols(p_addr + 32 * h, pk);
            }
            const float2 ps = fadd2(fadd2(part[0], part[1]), fadd2(part[2], part[3]));
            l = l * alpha + (ps.x + ps.y);
            m = m_new;
            // the rows whose maximum moved take O_i down by alpha (O_i holds
            // blocks 0 .. j-1, so PV_i(j - 1) has to be complete)
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                if (!CF::SEPARATE_P && !(ok = wait_warp(CF::BAR_PV + tile, jp ^ 1u)))
                    break;
                tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_load_32cols(o_addr + 32 * c, o);
                    tmem_load_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_store_32cols(o_addr + 32 * c, o);
                }
            }
            tmem_store_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(CF::BAR_PF + tile));
        }
        // output: O_i / l once the last P V has landed
        if (ok && nb > 0)
            ok = wait_warp(CF::BAR_PV + tile, static_cast<uint32_t>(nb - 1) & 1u);
        if (ok && nb > 0) {
            tc_fence_after_sync();
            const float inv = 1.0f / l;
            uint16_t *orow = p.O + (static_cast<size_t>(bh) * p.Sq + row) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_load_32cols(o_addr + 32 * c, o);
                tmem_load_wait();
                if (row < p.Sq && check_ok(static_cast<size_t>(bh) * p.Sq + row < static_cast<size_t>(p.BH) * p.Sq)) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack2<DT>(__uint_as_float(o[8 * v]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = pack2<DT>(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = pack2<DT>(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = pack2<DT>(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                        reinterpret_cast<uint4 *>(orow + 32 * c)[v] = w;
                    }
                }
            }
            if (p.lse && row < p.Sq)
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
