// attention_pair_kernel.cuh -- attention forward for head_dim 128 on a CTA
// pair (cluster of two), two query tiles per CTA in ping-pong:
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
// The pair computes four 128-row query tiles of one (batch, head), 512
// consecutive rows: CTA r holds tiles t = 0, 1 at rows q0 + 256 t + 128 r, so
// "pair tile" t is the 256 consecutive rows q0 + 256 t ... + 255, split
// between the two CTAs.  Every product is a cta_group::2 tcgen05.mma issued by
// the even CTA with M = 256: each CTA supplies its own 128 rows of the A
// operand and half of the B operand, and receives its own 128 rows of the
// result in its own Tensor Memory.  For each key block j of 128 keys:
//
//   S_t = Q_t K_j^T     A = Q_t (each CTA's rows), B = K_j: CTA r holds keys
//                       64 r .. 64 r + 63 of the block (all 128 head
//                       columns); S_t lands as 128 fp32 columns per CTA
//   P_t = 2^(S_t' - m)  each CTA's softmax warpgroup of tile t, one query row
//                       per thread, 16-bit weights written over S_t's first
//                       64 columns with tcgen05.st
//   O_t += P_t V_j      A = P_t read from Tensor Memory, B = V_j: CTA r holds
//                       head columns 64 r .. 64 r + 63 of all 128 keys
//
// so each CTA loads half of every K and V block, and each product moves twice
// the work of a single-CTA M = 128 product per instruction with half of the B
// operand read from each CTA's shared memory.  Issue order and the softmax are
// those of the single-CTA kernel: P V_0(j), S_0(j+1), P V_1(j), S_1(j+1); S
// waits for the P V it overwrites; the running maximum moves only when a row's
// new maximum exceeds it by more than 2^8, and then the warp rescales its rows
// of O in Tensor Memory.  Copies of both CTAs complete on the even CTA's
// barriers (which its MMA thread waits on); commits reach both CTAs; each
// softmax warp reports P ready on the even CTA's barrier.
//
// Warp roles (384 threads per CTA): warp 0 TMA producer, warp 1 TMEM allocator
// and (even CTA) MMA issuer, warps 2..3 idle, warps 4..7 softmax of tile 0,
// warps 8..11 softmax of tile 1.  Every wait is bounded; on expiry the kernel
// records it in the device error word, raises both CTAs' abort flags, lets
// issued copies and MMAs land (the even CTA drains the copies of both), frees
// TMEM and returns.
#pragma once

#include "attention_kernel.cuh"

namespace tl {

// 3-D tiled load into this CTA's shared memory whose byte count completes on
// an mbarrier that may live in the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map, uint32_t bar_cluster,
                                                 int32_t x, int32_t y, int32_t z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc] with M = 256 over the pair: each CTA's
// 128 rows of A in its own Tensor Memory, B split across the pair's shared
// memories at the same offsets; issued by the even CTA only.
__device__ __forceinline__ void tc_mma_f16_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                   uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int D_>
struct AttnPairConfig {
    static constexpr int D = D_;
    static constexpr int BM = 128, BN = 128, TILES = 2, CTAS = 2;
    static constexpr int ROWS = CTAS * TILES * BM;               // query rows per pair: 512
    static constexpr int KS = 4;                                 // K and V ring depth
    static constexpr int D_ATOMS = D / 64;
    static constexpr int Q_ATOM_BYTES = BM * 128;                // 128 rows x 64 16-bit values
    static constexpr int Q_BYTES = D_ATOMS * Q_ATOM_BYTES;       // one query tile
    static constexpr int KH_ROWS = BN / CTAS;                    // keys of a block this CTA holds
    static constexpr int K_ATOM_BYTES = KH_ROWS * 128;           // 64 keys x 64 head columns
    static constexpr int K_BYTES = D_ATOMS * K_ATOM_BYTES;       // this CTA's half of a K block
    static constexpr int V_BYTES = BN * 128;                     // 128 keys x this CTA's 64 head columns
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILES * Q_BYTES;
    static constexpr int OFF_V = OFF_K + KS * K_BYTES;
    static constexpr int OFF_BAR = OFF_V + KS * V_BYTES;
    static constexpr int BAR_Q = 0, BAR_KF = 1, BAR_KE = 1 + KS, BAR_VF = 1 + 2 * KS, BAR_VE = 1 + 3 * KS;
    static constexpr int BAR_SF = 1 + 4 * KS;   // [tile]: S_t(j) in Tensor Memory (both CTAs)
    static constexpr int BAR_PF = BAR_SF + 2;   // [tile]: P_t(j) written by all 8 softmax warps (even CTA)
    static constexpr int BAR_PV = BAR_PF + 2;   // [tile]: O_t += P_t(j) V_j completed (both CTAs)
    static constexpr int BAR_DRAIN = BAR_PV + 2;
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    // after the barriers: TMEM address, abort flag, 8 spare bytes, then the
    // copies issued per ring slot (Q, K[KS], V[KS]) by this CTA and by the odd CTA
    static constexpr int NUM_COUNTS = 1 + 2 * KS;
    static constexpr int OFF_COUNTS = OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr int SMEM_USED = OFF_COUNTS + 2 * NUM_COUNTS * 4;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;
    static constexpr int THREADS = 384;
    static constexpr int FIRST_SOFTMAX_WARP = 4;
    static constexpr int REGS_CONTROL = 64, REGS_SOFTMAX = 216;
    static constexpr int LAUNCH_REGS = (128 * REGS_CONTROL + 256 * REGS_SOFTMAX + THREADS - 1) / THREADS;
    static constexpr int TMEM_S = 0, TMEM_O = 256;  // S_t at 128 t, O_t at 256 + D t; P_t over S_t
    static constexpr float RESCALE_LOG2 = 8.0f;
    static_assert(D == 128, "the pair kernel is built for head_dim 128");
    static_assert(TMEM_O + TILES * D <= 512, "Tensor Memory columns");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <class CF, int DT>
__global__ void __launch_bounds__(384, 1)
    attention_pair_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                              const __grid_constant__ CUtensorMap tmap_v, const AttnParams p)
{
    constexpr int D = CF::D;
    constexpr int KS = CF::KS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the products
    const bool leader = rank == 0;

    // Pairs of CTAs along x.  Non-causal: 512-row query blocks along x, so the
    // pairs that start together share a head's K and V in L2.  Causal: heads
    // along x and the query blocks reversed along y, heaviest first.
    const int num_qblocks = (p.Sq + CF::ROWS - 1) / CF::ROWS;
    const int cx = static_cast<int>(blockIdx.x >> 1);
    const int qb = p.causal ? num_qblocks - 1 - static_cast<int>(blockIdx.y) : cx;
    const int bh = p.causal ? cx : static_cast<int>(blockIdx.y);
    const int q0 = qb * CF::ROWS;
    const int kblocks_all = (p.Sk + CF::BN - 1) / CF::BN;
    // key blocks pair tile t visits: its 256 rows q0 + 256 t ... (none past the queries)
    auto blocks_of = [&](int t) {
        const int first = q0 + 2 * CF::BM * t;
        if (first >= p.Sq)
            return 0;
        return p.causal ? min(kblocks_all, (first + 2 * CF::BM - 1) / CF::BN + 1) : kblocks_all;
    };
    const int nb0 = blocks_of(0), nb1 = blocks_of(1);
    auto nbt = [&](int t) { return t ? nb1 : nb0; };
    const int nbmax = max(nb0, nb1);

    const uint32_t sQ = smem_addr(smem + CF::OFF_Q);
    const uint32_t sK = smem_addr(smem + CF::OFF_K);
    const uint32_t sV = smem_addr(smem + CF::OFF_V);
    const uint32_t bar0 = smem_addr(smem + CF::OFF_BAR);
    auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    auto bar_lead = [&](int i) { return mapa_shared(bar(i), 0); };  // the even CTA's barrier i
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CF::OFF_BAR + CF::NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t peer_abort = mapa_shared(smem_addr(tmem_slot + 1), rank ^ 1u);
    // copies issued per ring slot [Q, K 0..KS-1, V 0..KS-1]: this CTA's, then (on the even CTA) the odd CTA's
    volatile uint32_t *issue_count = reinterpret_cast<volatile uint32_t *>(smem + CF::OFF_COUNTS);
    volatile uint32_t *peer_issue_count = issue_count + CF::NUM_COUNTS;

    if (threadIdx.x == 0) {
        mbar_init(bar(CF::BAR_Q), 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(bar(CF::BAR_KF + s), 1);
            mbar_init(bar(CF::BAR_KE + s), 1);
            mbar_init(bar(CF::BAR_VF + s), 1);
            mbar_init(bar(CF::BAR_VE + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(CF::BAR_SF + t), 1);
            mbar_init(bar(CF::BAR_PF + t), 4 * CF::CTAS);
            mbar_init(bar(CF::BAR_PV + t), 1);
        }
        mbar_init(bar(CF::BAR_DRAIN), 1);
        *abort_flag = 0;
        for (int s = 0; s < 2 * CF::NUM_COUNTS; ++s)
            issue_count[s] = 0u;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmap_q);
        tma_prefetch_map(&tmap_k);
        tma_prefetch_map(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(tmem_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();  // both CTAs' barriers and Tensor Memory exist before any cross-CTA use
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t timeout = p.timeout_ns;
    grid_dependency_wait();
    grid_launch_dependents();

    if (warp < CF::FIRST_SOFTMAX_WARP) {
        regs_decrease<CF::REGS_CONTROL>();
        if (warp == 0) {
            // ------------------------------------------------------------ producer (both CTAs)
            if (lane == 0) {
                bool ok = true;
                // both CTAs' query tiles complete on the even CTA's barrier
                if (leader)
                    mbar_arrive_expect_tx(bar(CF::BAR_Q), CF::CTAS * CF::TILES * CF::Q_BYTES);
#pragma unroll
                for (int t = 0; t < CF::TILES; ++t)
#pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d_pair(sQ + t * CF::Q_BYTES + a * CF::Q_ATOM_BYTES, &tmap_q, bar_lead(CF::BAR_Q),
                                         64 * a, q0 + 2 * CF::BM * t + CF::BM * static_cast<int>(rank), bh);
                issue_count[0] = 1u;
                int st = 0;
                uint32_t ph = 0;
                for (int j = 0; ok && j < nbmax; ++j) {
                    if (!wait_bounded<true>(bar(CF::BAR_KE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER,
                                            peer_abort)) {
                        ok = false;
                        break;
                    }
                    if (leader)
                        mbar_arrive_expect_tx(bar(CF::BAR_KF + st), CF::CTAS * CF::K_BYTES);
#pragma unroll
                    for (int a = 0; a < CF::D_ATOMS; ++a)
                        tma_load_3d_pair(sK + st * CF::K_BYTES + a * CF::K_ATOM_BYTES, &tmap_k, bar_lead(CF::BAR_KF + st),
                                         64 * a, j * CF::BN + CF::KH_ROWS * static_cast<int>(rank), bh);
                    issue_count[1 + st] = issue_count[1 + st] + 1u;
                    if (!wait_bounded<true>(bar(CF::BAR_VE + st), ph ^ 1u, abort_flag, timeout, ERR_PRODUCER,
                                            peer_abort)) {
                        ok = false;
                        break;
                    }
                    if (leader)
                        mbar_arrive_expect_tx(bar(CF::BAR_VF + st), CF::CTAS * CF::V_BYTES);
                    tma_load_3d_pair(sV + st * CF::V_BYTES, &tmap_v, bar_lead(CF::BAR_VF + st),
                                     64 * static_cast<int>(rank), j * CF::BN, bh);
                    issue_count[1 + KS + st] = issue_count[1 + KS + st] + 1u;
                    if (++st == KS) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer (even CTA)
            if (lane == 0 && leader) {
                constexpr uint32_t IDESC_QK = mma_idesc_f16(DT, 256, CF::BN, 0, 0);  // Q, K both K-major
                constexpr uint32_t IDESC_PV = mma_idesc_f16(DT, 256, D, 0, 1);       // P K-major (TMEM), V N-major
                const uint64_t k_desc0 = smem_desc_sw128(sK, 16, 1024);
                const uint64_t v_desc0 = smem_desc_sw128(sV, CF::V_BYTES, 1024);
                // K-major operands, K step k of 16: atom k / 4, +32 B inside it
                auto kmaj_q = [](int k) {
                    return static_cast<uint64_t>(((k >> 2) * CF::Q_ATOM_BYTES + (k & 3) * 32) >> 4);
                };
                auto kmaj_k = [](int k) {
                    return static_cast<uint64_t>(((k >> 2) * CF::K_ATOM_BYTES + (k & 3) * 32) >> 4);
                };
                int kst = 0, vst = 0;
                uint32_t kph = 0, vph = 0;
                bool ok = wait_bounded<true>(bar(CF::BAR_Q), 0, abort_flag, timeout, ERR_MMA_DATA, peer_abort);
                auto issue_s = [&](int t) {  // S_t = Q_t K^T from the current K slot
                    const uint64_t q_desc = smem_desc_sw128(sQ + t * CF::Q_BYTES, 16, 1024);
                    const uint64_t kd = k_desc0 + ((kst * CF::K_BYTES) >> 4);
                    const uint32_t d_s = tmem_base + static_cast<uint32_t>(CF::TMEM_S + t * 128);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_mma_f16_pair(d_s, q_desc + kmaj_q(k), kd + kmaj_k(k), IDESC_QK, k != 0 ? 1u : 0u);
                    tc_commit_pair_mc(bar(CF::BAR_SF + t), 0x3);
                };
                auto issue_pv = [&](int t, int j) {  // O_t (+)= P_t V from the current V slot
                    const uint32_t d_o = tmem_base + static_cast<uint32_t>(CF::TMEM_O + t * D);
                    const uint32_t a_p = tmem_base + static_cast<uint32_t>(CF::TMEM_S + t * 128);
                    const uint64_t vd = v_desc0 + ((vst * CF::V_BYTES) >> 4);
#pragma unroll
                    for (int k = 0; k < CF::BN / 16; ++k)  // 16 keys: 8 columns of P, 2048 B down V
                        tc_mma_f16_ts_pair(d_o, a_p + 8 * k, vd + ((2048 * k) >> 4), IDESC_PV,
                                           (j > 0 || k > 0) ? 1u : 0u);
                    tc_commit_pair_mc(bar(CF::BAR_PV + t), 0x3);
                };
                // prologue: S_0(0), S_1(0)
                if (ok && nbmax > 0) {
                    ok = wait_bounded<true>(bar(CF::BAR_KF + kst), kph, abort_flag, timeout, ERR_MMA_DATA, peer_abort);
                    if (ok) {
                        tc_fence_after_sync();
                        for (int t = 0; t < 2; ++t)
                            if (nbt(t) > 0)
                                issue_s(t);
                        tc_commit_pair_mc(bar(CF::BAR_KE + kst), 0x3);
                        if (++kst == KS) {
                            kst = 0;
                            kph ^= 1u;
                        }
                    }
                }
                for (int j = 0; ok && j < nbmax; ++j) {
                    const uint32_t jp = static_cast<uint32_t>(j) & 1u;
                    bool k_ready = false;  // K(j + 1) waited for
                    if (!wait_bounded<true>(bar(CF::BAR_VF + vst), vph, abort_flag, timeout, ERR_MMA_DATA, peer_abort)) {
                        ok = false;
                        break;
                    }
                    for (int t = 0; ok && t < 2; ++t) {
                        if (j < nbt(t)) {
                            if (!wait_bounded<true>(bar(CF::BAR_PF + t), jp, abort_flag, timeout, ERR_MMA_DATA,
                                                    peer_abort)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after_sync();
                            issue_pv(t, j);
                        }
                        if (t == 1)
                            tc_commit_pair_mc(bar(CF::BAR_VE + vst), 0x3);  // V(j) free once the last P V of block j is done
                        if (j + 1 < nbt(t)) {
                            // S_t(j + 1) overwrites the P_t(j) that P V_t(j) reads: wait for it
                            if ((!k_ready && !wait_bounded<true>(bar(CF::BAR_KF + kst), kph, abort_flag, timeout,
                                                                 ERR_MMA_DATA, peer_abort)) ||
                                !wait_bounded<true>(bar(CF::BAR_PV + t), jp, abort_flag, timeout, ERR_MMA_ACC,
                                                    peer_abort)) {
                                ok = false;
                                break;
                            }
                            k_ready = true;
                            tc_fence_after_sync();
                            issue_s(t);
                        }
                    }
                    if (!ok)
                        break;
                    if (++vst == KS) {
                        vst = 0;
                        vph ^= 1u;
                    }
                    if (k_ready) {
                        tc_commit_pair_mc(bar(CF::BAR_KE + kst), 0x3);
                        if (++kst == KS) {
                            kst = 0;
                            kph ^= 1u;
                        }
                    }
                }
                // every product issued above completes before Tensor Memory is released
                tc_commit_pair_mc(bar(CF::BAR_DRAIN), 0x1);
                wait_drain(bar(CF::BAR_DRAIN), 0, timeout);
            }
            __syncwarp();
        }
    } else {
        regs_increase<CF::REGS_SOFTMAX>();
        // ------------------------------------------------------------ softmax and output of one tile (both CTAs)
        const int tile = (warp - CF::FIRST_SOFTMAX_WARP) >> 2;
        const int q = warp & 3;
        const int r = q * 32 + lane;                                                   // row of the tile (TMEM lane)
        const int row = q0 + 2 * CF::BM * tile + CF::BM * static_cast<int>(rank) + r;  // query index
        const int nb = nbt(tile);
        // checked build: this tile's Tensor Memory columns inside the 512
        // allocated, its key blocks inside K
        check_ok(CF::TMEM_S + tile * 128 + 128 <= 512 && CF::TMEM_O + tile * D + D <= 512 && nb <= kblocks_all &&
                 bh < p.BH);
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t s_addr = tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_S + tile * 128);
        const uint32_t p_addr = s_addr;
        const uint32_t o_addr = tmem_base + lane_base + static_cast<uint32_t>(CF::TMEM_O + tile * D);
        auto wait_warp = [&](int id, uint32_t parity) -> bool {
            const bool w = wait_bounded<true>(bar(id), parity, abort_flag, timeout, ERR_EPILOGUE, peer_abort);
            return __all_sync(0xffffffffu, w);
        };
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
            // the rows whose maximum moved take O_t down by alpha (O_t holds
            // blocks 0 .. j-1, so P V_t(j - 1) has to be complete)
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                if (!(ok = wait_warp(CF::BAR_PV + tile, jp ^ 1u)))
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
                mbar_arrive_cluster(bar_lead(CF::BAR_PF + tile));
        }
        // output: O_t / l once the last P V has landed
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
    // The odd CTA's copies complete on the even CTA's barriers: hand it this
    // CTA's per-slot copy counts, so that it can drain for both.
    if (!leader && warp == 0 && lane == 0) {
        for (int s = 0; s < CF::NUM_COUNTS; ++s)
            st_shared_cluster_u32(mapa_shared(smem_addr(const_cast<uint32_t *>(peer_issue_count + s)), 0),
                                  issue_count[s]);
    }
    cluster_sync();
    if (leader && warp == 0 && lane == 0 && *abort_flag) {
        // Some role gave up: copies no one consumed may still be landing.  A
        // slot's copy is issued only after its previous contents were
        // consumed, so only the last phase of each slot can be pending; where
        // only one CTA issued that phase, complete the half that will never
        // come and wait for the half in flight.
        for (int s = 0; s < CF::NUM_COUNTS; ++s) {
            const uint32_t fb = s == 0 ? bar(CF::BAR_Q) : s <= KS ? bar(CF::BAR_KF + s - 1) : bar(CF::BAR_VF + s - 1 - KS);
            const uint32_t half = s == 0 ? CF::TILES * CF::Q_BYTES : s <= KS ? CF::K_BYTES : CF::V_BYTES;
            const uint32_t mine = issue_count[s], peer = peer_issue_count[s];
            const uint32_t n = mine > peer ? mine : peer;
            if (n == 0)
                continue;
            if (mine + 1 < n || peer + 1 < n) {
                atomicOr(&g_device_error, ERR_DRAIN);  // cannot happen: the counts differ by one at most
                continue;
            }
            if (mine == n && peer + 1 == n)
                mbar_complete_tx(fb, half);
            else if (peer == n && mine + 1 == n)
                mbar_arrive_expect_tx(fb, half);
            wait_drain(fb, (n - 1) & 1u, timeout);
        }
    }
    cluster_sync();  // the even CTA's products write this CTA's Tensor Memory and read its shared memory
    tc_fence_after_sync();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, 512);
}

} // namespace tl
