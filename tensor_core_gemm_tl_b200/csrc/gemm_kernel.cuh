// gemm_kernel.cuh -- persistent, warp-specialised sm_100a GEMM with a fused
// epilogue:  C = epilogue(A . B), epilogue = optional per-column bias, then
// optional GELU (exact erf form or tanh form); C 16-bit or float32.
//
// What it computes follows "Designing High-Performance GPU Kernels with
// TileLang" (blog retelling), Step 4 (tiled Tensor-Core GEMM: A tiles
// block_M x block_K and B tiles block_K x block_N staged through shared memory
// in a pipelined K loop, float32 accumulator) and the TileLang GPU kernel
// design article, paragraph 5 (bias add and GELU applied to the accumulator
// before the single store of C).  The pages' schedule (128/128/32, 2 stages,
// register fragments, mma.sync class) targets T4/A100/L4; on sm_100a the same
// roles map to:
//
//   global --TMA (128B swizzle)--> STAGES-deep shared-memory ring
//          --tcgen05.mma (one thread)--> fp32 accumulator in Tensor Memory
//          --tcgen05.ld--> registers: + bias, GELU, round once to fp16/bf16
//          --st.shared (swizzled)--> TMA store --> global
// (element stores when C's rows are not 16-byte aligned; with float32 C the
// fp32 values go straight out in 16-byte stores)
//
// Warp roles (320 threads, one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer (the whole warp walks the loop, one elected lane issues)
//   warp 1      TMEM allocator + MMA issuer (likewise)
//   warps 2..9  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31 and every
//               other 64-column chunk of them (two warps per lane quarter)
//
// Two TMEM accumulators (2 x BN fp32 columns) let the epilogue of tile i run
// while the MMAs of tile i+1 accumulate.  Every wait is bounded by a
// %globaltimer limit: on expiry the kernel records which wait gave up in a
// device error word, lets its issued copies and MMAs land (with a CTA pair,
// the even CTA drains the copies of both), frees TMEM and returns (no trap,
// no hang).  The last round of tiles can be cut along K across units; the
// parts of a tile are combined by whichever unit finishes last, so no unit
// ever waits for another.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100.cuh"

namespace tl {

// Device error word, read and cleared by tl_check_device.  This header is
// included by exactly one translation unit (tl_gemm.cu), which owns it.
__device__ unsigned int g_device_error = 0;

enum : unsigned {
    ERR_PRODUCER = 1u,
    ERR_MMA_DATA = 2u,
    ERR_MMA_ACC = 4u,
    ERR_EPILOGUE = 8u,
    ERR_DRAIN = 16u,
    ERR_SPLIT = 32u,   // a part of a split tile could not record its arrival (C incomplete)
    ERR_CHECK = 128u,  // checked build only: an index invariant failed (the access was skipped)
};

// The checked build (compiled with -DTL_CHECKED, libtlgemm_checked.so) tests
// the kernel's index invariants at run time: a violation sets ERR_CHECK in the
// device error word and the access it guards is skipped, never a trap.  In
// the product build check_ok() is the constant true and costs nothing.
#ifdef TL_CHECKED
constexpr bool kCheckedBuild = true;
#else
constexpr bool kCheckedBuild = false;
#endif

__device__ __forceinline__ bool check_ok(bool cond)
{
    if (kCheckedBuild && !cond) {
        atomicOr(&g_device_error, ERR_CHECK);
        return false;
    }
    return true;
}

struct GemmParams {
    int32_t M, N, K;
    int32_t tiles_m, tiles_n, num_tiles, num_kb;
    int32_t group_m;         // output-tile rows per rasterisation group
    const uint16_t *bias;    // N values of the input dtype (epilogue only)
    int32_t epi_bias;        // fused epilogue: add bias[col]
    int32_t epi_gelu;        // fused epilogue: 0 no GELU, 1 exact (erf) GELU, 2 tanh-form GELU
    int32_t bias_vec16;      // bias is 16-byte aligned: load 8 values per access
    int32_t inject_fault;    // test hook: every producer skips its first stage
    uint16_t *C;             // 16-bit element-store path only
    float *C32;              // float32 output only
    int32_t c32_vec16;       // float32 output: base 16-byte aligned and ldc % 4 == 0
    int64_t ldc;             // element-store and float32 paths (elements)
    uint64_t timeout_ns;
    // Work: tiles [0, full_tiles) whole, dealt round-robin to the units (CTAs,
    // or CTA pairs); then the `tail_tiles` tiles of the last round, whose
    // tail_tiles * num_kb k-blocks are cut into `tail_units` consecutive
    // ranges, one per unit.  A tile whose k-blocks fall to several units is
    // finished by whichever of them arrives last: each writes its fp32 partial
    // sums to its own slot of `partials` and then counts itself on the tile's
    // arrival word (tagged with this launch's `epoch`); the unit that completes
    // the count adds the parts in k order and runs the epilogue.  No unit ever
    // waits for another.
    int32_t full_tiles, tail_tiles, tail_units;
    int32_t num_slots;       // partial-sum slots in the workspace (tail_units + tail_tiles - 1)
    float *partials;         // [slot][cta of the pair][lane quarter][64-column chunk][16 float4][32 lanes]
    unsigned long long *arrivals;  // [tail tile][cta][lane quarter][warp of the quarter]
    unsigned long long epoch;  // unique per launch, below 2^56
};

// One unit of work: k-blocks [kb0, kb1) of output tile `tile`.  `tail` is the
// tile's index in the last round when its k-blocks are cut across units (else
// -1).
struct WorkItem {
    int tile, kb0, kb1, tail;
};

// What one unit computes: n_full whole tiles (unit, unit + num_units, ...),
// then up to two pieces of the last round (its k-block range can end in the
// next tile).
struct UnitWork {
    int n_full, n_seg;
    int seg_r0, seg_kb00, seg_kb10;
    int seg_r1, seg_kb01, seg_kb11;
};

__device__ __forceinline__ UnitWork unit_work(int unit, int num_units, const GemmParams &p)
{
    UnitWork u{};
    u.n_full = unit < p.full_tiles ? (p.full_tiles - 1 - unit) / num_units + 1 : 0;
    u.n_seg = 0;
    if (unit < p.tail_units) {
        const int64_t T = static_cast<int64_t>(p.tail_tiles) * p.num_kb;
        int64_t g = static_cast<int64_t>(unit) * T / p.tail_units;
        const int64_t g1 = static_cast<int64_t>(unit + 1) * T / p.tail_units;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (g >= g1)
                break;
            const int r = static_cast<int>(g / p.num_kb);
            const int64_t base = static_cast<int64_t>(r) * p.num_kb;
            const int64_t end = g1 < base + p.num_kb ? g1 : base + p.num_kb;
            if (i == 0) {
                u.seg_r0 = r;
                u.seg_kb00 = static_cast<int>(g - base);
                u.seg_kb10 = static_cast<int>(end - base);
            } else {
                u.seg_r1 = r;
                u.seg_kb01 = static_cast<int>(g - base);
                u.seg_kb11 = static_cast<int>(end - base);
            }
            u.n_seg = i + 1;
            g = end;
        }
    }
    return u;
}

__device__ __forceinline__ WorkItem work_item(const UnitWork &u, int i, int unit, int num_units,
                                              const GemmParams &p)
{
    WorkItem w;
    if (i < u.n_full) {
        w.tile = unit + i * num_units;
        w.kb0 = 0;
        w.kb1 = p.num_kb;
        w.tail = -1;
    } else {
        const bool second = i > u.n_full;
        w.tail = second ? u.seg_r1 : u.seg_r0;
        w.tile = p.full_tiles + w.tail;
        w.kb0 = second ? u.seg_kb01 : u.seg_kb00;
        w.kb1 = second ? u.seg_kb11 : u.seg_kb10;
    }
    return w;
}

// The units whose k-block ranges meet tail tile r: first .. last.  Unit u's
// range starts at floor(u T / U), so the unit holding global k-block x is
// ceil((x + 1) U / T) - 1 (T tail k-blocks, U tail units).
__device__ __forceinline__ void tail_contributors(int r, const GemmParams &p, int &first, int &last)
{
    const int64_t T = static_cast<int64_t>(p.tail_tiles) * p.num_kb;
    const int64_t U = p.tail_units;
    const int64_t x0 = static_cast<int64_t>(r) * p.num_kb;
    const int64_t x1 = x0 + p.num_kb - 1;
    first = static_cast<int>(((x0 + 1) * U + T - 1) / T) - 1;
    last = static_cast<int>(((x1 + 1) * U + T - 1) / T) - 1;
}

// Count one more part of a split tile on its arrival word and return the
// count (0 if the word could not be updated, which is recorded).  The word's
// upper 56 bits hold the launch's epoch: a word that carries another epoch
// (left by an earlier launch, or never written) counts as zero.
__device__ __forceinline__ unsigned arrive_tagged(unsigned long long *word, unsigned long long epoch)
{
    const unsigned long long tag = epoch << 8;
    unsigned long long old = ld_relaxed_u64(word);
    for (int i = 0; i < 4096; ++i) {
        const unsigned long long next = (old & ~0xFFull) == tag ? old + 1ull : (tag | 1ull);
        const unsigned long long seen = atom_cas_acq_rel_u64(word, old, next);
        if (seen == old)
            return static_cast<unsigned>(next & 0xFFull);
        old = seen;
    }
    atomicOr(&g_device_error, ERR_SPLIT);
    return 0u;
}

// Compile-time tile configuration.  Each CTA owns BM = 128 output rows (one
// TMEM lane per row) and BK = 64 (one 128-byte swizzle row of 16-bit values).
// PAIR = false: one CTA computes a 128 x BN tile with cta_group::1 MMAs.
// PAIR = true:  a cluster of two CTAs computes a 256 x BN tile with
//               cta_group::2 MMAs issued by the even CTA; each CTA loads its
//               own 128 rows of A and its own BN/2 columns of B, and holds its
//               128 rows of the accumulator in its own TMEM.
template <int BN_, int STAGES_, bool PAIR_ = false>
struct TileConfig {
    static constexpr bool PAIR = PAIR_;
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int BM = 128, BN = BN_, BK = 64, STAGES = STAGES_;
    static constexpr int TILE_M = BM * CTAS;       // output rows per tile
    static constexpr int BN_LOCAL = BN / CTAS;     // B columns this CTA loads
    static constexpr int A_STAGE_BYTES = BM * BK * 2;
    static constexpr int B_BOX_BYTES = BK * 128;   // one 64-column box of B
    static constexpr int B_STAGE_BYTES = BK * BN_LOCAL * 2;
    static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
    static constexpr int TX_BYTES = STAGE_BYTES * CTAS;  // landing on the (even CTA's) full barrier
    // two epilogue warps per TMEM lane quarter; they split the 64-column chunks
    static constexpr int EPI_WARPS = 8;
    static constexpr int C_BOX_BYTES = 32 * 128;   // 32 rows x 64 columns of 16-bit
    static constexpr int C_STAGING_BYTES = EPI_WARPS * C_BOX_BYTES;  // one box per epilogue warp
    static constexpr int ACC_COLS = BN;             // fp32 TMEM columns per accumulator
    static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_STAGE_BYTES;
    static constexpr int OFF_C = OFF_B + STAGES * B_STAGE_BYTES;
    static constexpr int OFF_BAR = OFF_C + C_STAGING_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 5;
    // after the barriers: TMEM address, abort flag, 8 spare bytes, then the
    // copies issued per stage by this CTA and (pair) by the odd CTA
    static constexpr int OFF_COUNTS = OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr int SMEM_USED = OFF_COUNTS + 2 * STAGES * 4;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;  // producer, MMA, epilogue warps
    static_assert(BN_LOCAL % 64 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM columns");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Output tile t -> (tile row, tile col), grouped so that consecutive tiles
// share A rows within a group of `group_m` tile rows (L2 reuse).
__device__ __forceinline__ void tile_coords(int t, const GemmParams &p, int &tm, int &tn)
{
    const int group_size = p.group_m * p.tiles_n;
    const int g = t / group_size;
    const int first_m = g * p.group_m;
    const int rows = min(p.tiles_m - first_m, p.group_m);
    const int r = t - g * group_size;
    tm = first_m + r % rows;
    tn = r / rows;
}

// Bounded wait.  Returns false when the abort flag is raised by another role
// (or by the peer CTA) or when this wait runs past timeout_ns; then it raises
// the flag itself, and the peer's too when `peer_abort` (a shared::cluster
// address) is non-zero.  CLUSTER_SCOPE acquires at cluster scope, for
// barriers the peer CTA arrives on.
template <bool CLUSTER_SCOPE = false>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             uint64_t timeout_ns, unsigned code, uint32_t peer_abort = 0)
{
    auto test = [&]() { return CLUSTER_SCOPE ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
    if (test())
        return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (test())
            return true;
        if (*abort_flag)
            return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1;
            if (peer_abort)
                st_shared_cluster_u32(peer_abort, 1u);
            atomicOr(&g_device_error, code);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (used to let in-flight work land).
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > timeout_ns) {
            atomicOr(&g_device_error, ERR_DRAIN);
            return false;
        }
    }
    return true;
}

template <int DT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (DT == 1) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

template <int DT>
__device__ __forceinline__ float to_float(uint16_t bits)
{
    if constexpr (DT == 1)
        return __uint_as_float(static_cast<uint32_t>(bits) << 16);
    else
        return __half2float(__ushort_as_half(bits));
}

// Exact GELU on the fp32 accumulator: x * Phi(x), Phi the standard normal CDF.
//   z = |x| / sqrt 2,  Phi(x) = 1 - erfc(z)/2 (x >= 0),  erfc(z)/2 (x < 0)
//   erfc(z) = exp(-z^2) h(t),  t = 1 / (1 + p z)
// The substitution t is that of Abramowitz & Stegun, Handbook of Mathematical
// Functions, 7.1.26; h is this library's own degree-8 least-squares fit to
// exp(z^2) erfc(z) on z in [0, 9.25] (relative error of h ~3e-8; the
// coefficients come from csrc/fit_gelu_erfcx.py).  exp(-z^2) = 2^(-x^2 log2(e) / 2)
// is taken from x^2 split exactly into hi + lo (one fma), so the argument does
// not lose the low bits of x^2 and loses only the rounding of one product as |x| grows.  Computing erfc of |x|
// avoids the cancellation of 1 + erf(x / sqrt 2) for negative x.  Relative
// error below 3e-6 for |x| <= 9 (below 1e-5 everywhere; one fp16 ulp is 5e-4,
// one bf16 ulp 4e-3); NaN stays NaN.
// Both GELU forms run on pairs of values: their multiply-adds take two lanes
// per instruction (fma/mul/add .f32x2, each lane rounded as its scalar step).
__device__ __forceinline__ float2 gelu_erf2(float2 x)
{
    constexpr float P_SQRT1_2 = 0.415f * 0.70710678118654752f;
    constexpr float C0 = 4.281122892280109e-05f, C1 = 0.23316948115825653f, C2 = 0.24358120560646057f,
                    C3 = 0.1621198058128357f, C4 = 0.34987202286720276f, C5 = -0.2624722123146057f,
                    C6 = 0.5700822472572327f, C7 = -0.3758394122123718f, C8 = 0.079444020986557f;
    constexpr float NEG_HALF_LOG2E = -0.72134752044448170f;
    const float2 a = make_float2(fminf(fabsf(x.x), 20.0f), fminf(fabsf(x.y), 20.0f));
    const float2 d = ffma2(splat2(P_SQRT1_2), a, splat2(1.0f));
    const float2 t = make_float2(rcp_approx(d.x), rcp_approx(d.y));
    float2 h = ffma2(splat2(C8), t, splat2(C7));
    h = ffma2(h, t, splat2(C6));
    h = ffma2(h, t, splat2(C5));
    h = ffma2(h, t, splat2(C4));
    h = ffma2(h, t, splat2(C3));
    h = ffma2(h, t, splat2(C2));
    h = ffma2(h, t, splat2(C1));
    h = ffma2(h, t, splat2(C0));
    const float2 hi = fmul2(a, a);
    const float2 lo = ffma2(a, a, make_float2(-hi.x, -hi.y));
    const float2 m = fmul2(hi, splat2(NEG_HALF_LOG2E));
    const float2 e = fmul2(make_float2(exp2_approx(m.x), exp2_approx(m.y)), ffma2(splat2(-0.5f), lo, splat2(1.0f)));
    const float2 q = fmul2(fmul2(splat2(0.5f), h), e);
    const float2 one_q = fadd2(splat2(1.0f), make_float2(-q.x, -q.y));
    return fmul2(x, make_float2(x.x >= 0.0f ? one_q.x : q.x, x.y >= 0.0f ? one_q.y : q.y));
}

// Tanh form of GELU (the GELU paper's approximation):
//     g(x) = 0.5 x (1 + tanh(u)),   u = sqrt(2 / pi) (x + 0.044715 x^3),
// through 0.5 (1 + tanh u) = 1 / (1 + 2^-a) for x >= 0 and 2^-a / (1 + 2^-a)
// for x < 0, a = |2u| log2(e): the exponential never exceeds 1, so nothing
// overflows or cancels.  u has the sign of x.  Relative error about
// 3e-7 + 1.2e-7 a (the rounding of a, carried through 2^-a): below 1e-5
// for x >= -10, where g is 1e-37.  NaN stays NaN.
__device__ __forceinline__ float2 gelu_tanh2(float2 x)
{
    constexpr float K0 = 2.3022081983f;
    constexpr float K1 = 0.044715f * K0;
    const float2 inner = ffma2(splat2(K1), fmul2(x, x), splat2(K0));
    const float2 a = fmul2(make_float2(fabsf(x.x), fabsf(x.y)), inner);
    const float2 e = make_float2(exp2_approx(-a.x), exp2_approx(-a.y));
    const float2 den = fadd2(splat2(1.0f), e);
    const float2 s = make_float2(rcp_approx(den.x), rcp_approx(den.y));
    const float2 es = fmul2(e, s);
    return fmul2(x, make_float2(x.x >= 0.0f ? s.x : es.x, x.y >= 0.0f ? s.y : es.y));
}

// How C leaves the epilogue.
enum StoreMode : int {
    STORE_ELEMENTS = 0,  // 16-bit C, element stores (rows not 16-byte aligned)
    STORE_TMA = 1,       // 16-bit C, swizzled shared-memory staging and TMA stores
    STORE_F32 = 2,       // float32 C (no rounding to 16 bits), vector or element stores
};

// EPI = 0: C = A.B.  EPI = 1: the fused epilogue, its steps chosen at run
// time (bias add and/or a GELU form).  BT: B is given as N x K row-major
// (K-major operand) instead of K x N.
template <class CF, int DT, int EPI, int STORE, bool BT>
__global__ void __launch_bounds__(CF::THREADS, 1)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_c, const GemmParams p)
{
    constexpr bool PAIR = CF::PAIR;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    // The warp index through a shuffle from lane 0: the compiler can then prove
    // it, and the role branches taken on it, uniform across the warp.
    const int warp = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0: the CTA that issues the MMAs
    const bool leader = rank == 0;
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int num_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    const uint32_t sA = smem_addr(smem + CF::OFF_A);
    const uint32_t sB = smem_addr(smem + CF::OFF_B);
    uint8_t *cstage = smem + CF::OFF_C;
    const uint32_t bar0 = smem_addr(smem + CF::OFF_BAR);
    // barrier i lives at bar0 + 8 i
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (CF::STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * CF::STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * CF::STAGES + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (2 * CF::STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + CF::OFF_BAR + CF::NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t peer_abort = PAIR ? mapa_shared(smem_addr(tmem_slot + 1), rank ^ 1u) : 0u;
    // copies issued per stage: by this CTA, and (on the even CTA of a pair) by the odd one
    volatile uint32_t *issue_count = reinterpret_cast<volatile uint32_t *>(smem + CF::OFF_COUNTS);
    volatile uint32_t *peer_issue_count = issue_count + CF::STAGES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), CF::EPI_WARPS * CF::CTAS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        for (int s = 0; s < 2 * CF::STAGES; ++s)
            issue_count[s] = 0u;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmap_a);
        tma_prefetch_map(&tmap_b);
        if constexpr (STORE == STORE_TMA)
            tma_prefetch_map(&tmap_c);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), CF::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), CF::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before_sync();
    if constexpr (PAIR)
        cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA use
    else
        __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const uint64_t timeout = p.timeout_ns;
    // Under the fault hook the copy and epilogue roles wait twice as long, so
    // that the wait which gives up first is always the MMA warp's wait on the
    // skipped stage (every role starts waiting within microseconds of the others).
    const uint64_t timeout_other = p.inject_fault ? 2 * timeout : timeout;
    // Everything above touches only this CTA's own state, so it may overlap the
    // previous kernel on the stream; global memory is read and written only
    // after that kernel has completed.  With CTA pairs every thread waits here.
    // Single CTAs wait role by role, just before each role's first global
    // access: the producer's set-up then runs while the previous kernel
    // finishes (measured: 3.5% on a 26 us HBM-bound launch; the same change
    // cost CTA-pair GEMMs 1.6%), and the MMA warp touches no global memory.
    if constexpr (PAIR)
        grid_dependency_wait();
    grid_launch_dependents();

    // Every role walks the same list of work items.
    const UnitWork uw = unit_work(unit, num_units, p);
    const int n_items = uw.n_full + uw.n_seg;
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the loop (its control flow and values are then
        // the same in every lane); one elected lane issues each stage's copies.
        // Measured against a loop run by lane 0 alone: 2-7% faster GEMMs, most
        // with the fused epilogue, whose warps share the producer's scheduler.
        {
            int stage = 0;
            uint32_t phase = 0;
            bool skip = p.inject_fault != 0;  // both CTAs of a pair skip the same stage
            bool ok = true;
            bool dep_wait = !PAIR;  // single CTAs: the previous kernel not yet waited for
            for (int i = 0; ok && i < n_items; ++i) {
                const WorkItem w = work_item(uw, i, unit, num_units, p);
                int tm, tn;
                tile_coords(w.tile, p, tm, tn);
                check_ok(w.tile < p.num_tiles && w.tail < p.tail_tiles && w.kb0 < w.kb1 && w.kb1 <= p.num_kb &&
                         tm < p.tiles_m && tn < p.tiles_n);  // TMA clips anything outside: record only
                const int a_row = tm * CF::TILE_M + static_cast<int>(rank) * CF::BM;
                const int b_col = tn * CF::BN + static_cast<int>(rank) * CF::BN_LOCAL;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!__all_sync(0xffffffffu, wait_bounded<PAIR>(empty_bar(stage), phase ^ 1u, abort_flag,
                                                                    timeout_other, ERR_PRODUCER, peer_abort))) {
                        ok = false;
                        break;
                    }
                    if (dep_wait) {
                        grid_dependency_wait();
                        dep_wait = false;
                    }
                    if (skip) {
                        skip = false;
                    } else if (elect_one()) {
                        const uint32_t fb = full_bar(stage);
                        const uint32_t sa = sA + stage * CF::A_STAGE_BYTES;
                        const uint32_t sb = sB + stage * CF::B_STAGE_BYTES;
                        if constexpr (PAIR) {
                            // both CTAs' bytes complete on the even CTA's barrier
                            const uint32_t fb0 = mapa_shared(fb, 0);
                            if (leader)
                                mbar_arrive_expect_tx(fb, CF::TX_BYTES);
                            tma_load_2d_pair(sa, &tmap_a, fb0, kb * CF::BK, a_row);
                            if constexpr (BT) {
                                tma_load_2d_pair(sb, &tmap_b, fb0, kb * CF::BK, b_col);  // BN_LOCAL rows of B^T
                            } else {
#pragma unroll
                                for (int j = 0; j < CF::BN_LOCAL / 64; ++j)
                                    tma_load_2d_pair(sb + j * CF::B_BOX_BYTES, &tmap_b, fb0, b_col + 64 * j,
                                                     kb * CF::BK);
                            }
                        } else {
                            mbar_arrive_expect_tx(fb, CF::TX_BYTES);
                            tma_load_2d(sa, &tmap_a, fb, kb * CF::BK, a_row);
                            if constexpr (BT) {
                                tma_load_2d(sb, &tmap_b, fb, kb * CF::BK, b_col);  // BN_LOCAL rows of B^T
                            } else {
#pragma unroll
                                for (int j = 0; j < CF::BN_LOCAL / 64; ++j)
                                    tma_load_2d(sb + j * CF::B_BOX_BYTES, &tmap_b, fb, b_col + 64 * j,
                                                kb * CF::BK);
                            }
                        }
                        issue_count[stage] = issue_count[stage] + 1u;
                    }
                    __syncwarp();
                    if (++stage == CF::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        // The whole warp walks the loop, so its control flow and every value it
        // computes are the same in all lanes; one elected lane (always the
        // same) issues each tcgen05 instruction.
        if (leader) {
            constexpr uint32_t IDESC = mma_idesc_f16(DT, CF::TILE_M, CF::BN, 0, BT ? 0 : 1);
            // A: K-major, rows of 128 B, 8-row atoms 1024 B apart (SBO); LBO unused.
            // B: N-major, 64-column boxes of BK rows (LBO = box bytes), 8-row atoms (SBO);
            //    or, given as B^T, K-major like A.
            const uint64_t a_desc0 = smem_desc_sw128(sA, 16, 1024);
            const uint64_t b_desc0 = BT ? smem_desc_sw128(sB, 16, 1024) : smem_desc_sw128(sB, CF::B_BOX_BYTES, 1024);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_items; ++i) {
                const WorkItem w = work_item(uw, i, unit, num_units, p);
                // every lane waits; the warp goes on only if all of them saw the phase
                if (!__all_sync(0xffffffffu, wait_bounded<PAIR>(tempty_bar(acc), acc_phase ^ 1u, abort_flag, timeout,
                                                                ERR_MMA_ACC, peer_abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * CF::ACC_COLS);
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!__all_sync(0xffffffffu, wait_bounded(full_bar(stage), phase, abort_flag, timeout,
                                                              ERR_MMA_DATA, peer_abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t a_desc = a_desc0 + ((stage * CF::A_STAGE_BYTES) >> 4);
                    const uint64_t b_desc = b_desc0 + ((stage * CF::B_STAGE_BYTES) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < CF::BK / 16; ++k) {
                            // K step of 16: +32 B inside A's swizzled row; B: +16 rows (2048 B),
                            // or +32 B when B is K-major
                            const uint64_t ad = a_desc + ((32 * k) >> 4);
                            const uint64_t bd = b_desc + (((BT ? 32 : 2048) * k) >> 4);
                            const uint32_t accumulate = (kb != w.kb0 || k != 0) ? 1u : 0u;
                            if constexpr (PAIR)
                                tc_mma_f16_pair(d_tmem, ad, bd, IDESC, accumulate);
                            else
                                tc_mma_f16(d_tmem, ad, bd, IDESC, accumulate);
                        }
                        if constexpr (PAIR)
                            tc_commit_pair_mc(empty_bar(stage), 0x3);
                        else
                            tc_commit(empty_bar(stage));
                    }
                    __syncwarp();
                    if (++stage == CF::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if (elect_one()) {
                    if constexpr (PAIR)
                        tc_commit_pair_mc(tfull_bar(acc), 0x3);
                    else
                        tc_commit(tfull_bar(acc));
                }
                __syncwarp();
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every MMA issued above completes before TMEM is released
            if (elect_one()) {
                if constexpr (PAIR)
                    tc_commit_pair_mc(drain_bar, 0x1);
                else
                    tc_commit(drain_bar);
            }
            __syncwarp();
            wait_drain(drain_bar, 0, timeout);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;               // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;     // which of the quarter's two warps: chunks c = half, half + 2, ...
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        constexpr int CHUNKS = CF::BN / 64;
        const int my_last = (CHUNKS - 1 - half) >= 0 ? half + 2 * ((CHUNKS - 1 - half) / 2) : -1;
        uint8_t *buf = cstage + (warp - 2) * CF::C_BOX_BYTES;
        int acc = 0;
        uint32_t acc_phase = 0;
        if constexpr (!PAIR)
            grid_dependency_wait();  // bias, C and the split's workspace
        for (int i = 0; i < n_items; ++i) {
            const WorkItem w = work_item(uw, i, unit, num_units, p);
            int tm, tn;
            tile_coords(w.tile, p, tm, tn);
            check_ok(w.tile < p.num_tiles && w.tail < p.tail_tiles && tm < p.tiles_m && tn < p.tiles_n);
            const int n0 = tn * CF::BN;
            // a tile of the last round whose k-blocks several units share
            int t_first = unit, t_last = unit;
            if (w.tail >= 0)
                tail_contributors(w.tail, p, t_first, t_last);
            const bool shared_tile = t_last > t_first;
            const int row0 = tm * CF::TILE_M + static_cast<int>(rank) * CF::BM + q * 32;  // this warp's rows
            if constexpr (EPI == 1) {
                // bring this warp's bias columns into L1 while the tile's
                // products run: the epilogue's bias loads then hit
                if (p.epi_bias && lane < CHUNKS) {
                    const int c = half + 2 * (lane >> 1);
                    const int col = n0 + c * 64 + (lane & 1) * 32;
                    if (c < CHUNKS && col < p.N)
                        prefetch_l1(p.bias + col);
                }
            }
            if (!wait_bounded<PAIR>(tfull_bar(acc), acc_phase, abort_flag, timeout_other, ERR_EPILOGUE,
                                    peer_abort))
                break;
            tc_fence_after_sync();
            auto release_accumulator = [&]() {
                // this warp's share of the accumulator is in registers: hand it back
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR)
                        mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
                    else
                        mbar_arrive(tempty_bar(acc));
                }
            };
            // Epilogue of one 32-row x 64-column chunk of C from its fp32 sums
            // (this warp's rows, columns col0 ..): + bias, GELU, one rounding,
            // store.
            auto store_chunk = [&](int c, uint32_t (&r)[64]) {
                const int col0 = n0 + c * 64;
                if constexpr (STORE == STORE_TMA) {
                    // this warp's staging box: its previous store must have read it
                    if (lane == 0)
                        bulk_wait_group_read<0>();
                    __syncwarp();
                }
                // two halves of 32 columns: fewer values live at once
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = __uint_as_float(r[32 * h + j]);
                    const int colh = col0 + 32 * h;
                    if constexpr (EPI == 1) {
                      if (p.epi_bias) {
                        if (p.bias_vec16 && colh + 32 <= p.N) {
                            const uint4 *bp = reinterpret_cast<const uint4 *>(p.bias + colh);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint4 w = __ldg(bp + i);
                                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 sum2 = fadd2(make_float2(v[8 * i + 2 * e], v[8 * i + 2 * e + 1]),
                                                              make_float2(to_float<DT>(static_cast<uint16_t>(ww[e] & 0xFFFFu)),
                                                                          to_float<DT>(static_cast<uint16_t>(ww[e] >> 16))));
                                    v[8 * i + 2 * e] = sum2.x;
                                    v[8 * i + 2 * e + 1] = sum2.y;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (colh + j < p.N)
                                    v[j] += to_float<DT>(__ldg(p.bias + colh + j));
                        }
                      }
                      if (p.epi_gelu == 1) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float2 g = gelu_erf2(make_float2(v[j], v[j + 1]));
                            v[j] = g.x;
                            v[j + 1] = g.y;
                        }
                      } else if (p.epi_gelu == 2) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float2 g = gelu_tanh2(make_float2(v[j], v[j + 1]));
                            v[j] = g.x;
                            v[j + 1] = g.y;
                        }
                      }
                    }
                    if constexpr (STORE == STORE_F32) {
                        // row `lane`: 32 consecutive floats (128 bytes)
                        const int m = row0 + lane;
                        if (m < p.M) {
                            float *crow = p.C32 + static_cast<int64_t>(m) * p.ldc + colh;
                            if (p.c32_vec16 && colh + 32 <= p.N) {
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    reinterpret_cast<float4 *>(crow)[i] =
                                        make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (colh + j < p.N)
                                        crow[j] = v[j];
                            }
                        }
                    } else {
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        packed[j] = pack2<DT>(v[2 * j], v[2 * j + 1]);
    
                    if constexpr (STORE == STORE_TMA) {
                        // row `lane` of the 32 x 64 box; 16-byte chunk i lands at i ^ (lane & 7)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int chunk = 4 * h + i;
                            *reinterpret_cast<uint4 *>(buf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                        }
                    } else {
                        const int m = row0 + lane;
                        if (m < p.M) {
                            uint16_t *crow = p.C + static_cast<int64_t>(m) * p.ldc;
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int n = colh + 2 * j;
                                if (n < p.N)
                                    crow[n] = static_cast<uint16_t>(packed[j] & 0xFFFFu);
                                if (n + 1 < p.N)
                                    crow[n + 1] = static_cast<uint16_t>(packed[j] >> 16);
                            }
                        }
                    }
                    }  // 16-bit C
                }
                if constexpr (STORE == STORE_TMA) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_c, smem_addr(buf), col0, row0);
                        bulk_commit_group();
                    }
                }
            };
            // Chunks this warp stores: c = half, half + 2, ... inside C.
            auto chunk_in_c = [&](int c) { return n0 + c * 64 < p.N && row0 < p.M; };
            if (my_last < 0)
                release_accumulator();
            if (!shared_tile) {
#pragma unroll 1
                for (int c = half; c < CHUNKS; c += 2) {
                    uint32_t r[64];
                    if (!check_ok(acc * CF::ACC_COLS + c * 64 + 64 <= CF::TMEM_COLS))
                        continue;  // outside this CTA's Tensor Memory
                    const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(acc * CF::ACC_COLS + c * 64);
                    tmem_load_32cols(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                    tmem_load_32cols(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                    tmem_load_wait();
                    if (c == my_last)
                        release_accumulator();
                    if (chunk_in_c(c))
                        store_chunk(c, r);
                }
            } else {
                // A tile of the split last round.  Every part writes its fp32
                // partial sums to its own slot, then counts itself on this
                // warp's arrival word (one per tail tile, CTA, lane quarter and
                // warp of the quarter); the part that completes the count adds
                // the parts in k order (first .. last unit, its own read back
                // like the others) and stores C.  A slot holds each warp's chunk
                // as 16 float4 columns of 32 lanes: every access is 512
                // contiguous bytes, and a part's chunk is read with all 16
                // loads in flight.
                const size_t slab_f4 = static_cast<size_t>(CF::BM) * CF::BN / 4;
                auto slot_f4 = [&](int u, int c) {
                    // slot u + r is unique per (unit, tail tile)
                    return reinterpret_cast<float4 *>(p.partials) +
                           (static_cast<size_t>(u + w.tail) * CF::CTAS + rank) * slab_f4 +
                           ((static_cast<size_t>(q) * CHUNKS + c) * 16) * 32 + lane;
                };
                const bool slots_ok = check_ok(static_cast<size_t>(t_last + w.tail) < static_cast<size_t>(p.num_slots));
                bool any = false;
#pragma unroll 1
                for (int c = half; c < CHUNKS; c += 2) {
                    uint32_t r[64];
                    if (!check_ok(acc * CF::ACC_COLS + c * 64 + 64 <= CF::TMEM_COLS))
                        continue;  // outside this CTA's Tensor Memory
                    const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(acc * CF::ACC_COLS + c * 64);
                    tmem_load_32cols(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                    tmem_load_32cols(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                    tmem_load_wait();
                    if (c == my_last)
                        release_accumulator();
                    if (!chunk_in_c(c) || !slots_ok)
                        continue;
                    any = true;
                    float4 *mine = slot_f4(unit, c);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        __stcg(mine + 32 * i, make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                          __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
                }
                if (any) {
                    // the warp's writes, then one release by lane 0 (the warp
                    // barrier orders the other lanes' writes before it)
                    __syncwarp();
                    unsigned count = 0;
                    if (lane == 0) {
                        const size_t word = ((static_cast<size_t>(w.tail) * CF::CTAS + rank) * 4 + q) * 2 + half;
                        fence_acq_rel_gpu();
                        count = arrive_tagged(p.arrivals + word, p.epoch);
                    }
                    count = __shfl_sync(0xffffffffu, count, 0);
                    if (count == static_cast<unsigned>(t_last - t_first + 1)) {
                        __syncwarp();  // lane 0's acquire orders the reads below
#pragma unroll 1
                        for (int c = half; c < CHUNKS; c += 2) {
                            if (!chunk_in_c(c))
                                continue;
                            uint32_t r[64];
                            {
                                const float4 *src = slot_f4(t_first, c);
#pragma unroll
                                for (int i = 0; i < 16; ++i) {
                                    const float4 a = __ldcg(src + 32 * i);
                                    r[4 * i] = __float_as_uint(a.x);
                                    r[4 * i + 1] = __float_as_uint(a.y);
                                    r[4 * i + 2] = __float_as_uint(a.z);
                                    r[4 * i + 3] = __float_as_uint(a.w);
                                }
                            }
#pragma unroll 1
                            for (int u = t_first + 1; u <= t_last; ++u) {
                                const float4 *src = slot_f4(u, c);
                                float4 b[16];
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    b[i] = __ldcg(src + 32 * i);
#pragma unroll
                                for (int i = 0; i < 16; ++i) {
                                    r[4 * i] = __float_as_uint(__uint_as_float(r[4 * i]) + b[i].x);
                                    r[4 * i + 1] = __float_as_uint(__uint_as_float(r[4 * i + 1]) + b[i].y);
                                    r[4 * i + 2] = __float_as_uint(__uint_as_float(r[4 * i + 2]) + b[i].z);
                                    r[4 * i + 3] = __float_as_uint(__uint_as_float(r[4 * i + 3]) + b[i].w);
                                }
                            }
                            store_chunk(c, r);
                        }
                    }
                }
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if constexpr (STORE == STORE_TMA) {
            if (lane == 0)
                bulk_wait_group<0>();
            __syncwarp();
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if constexpr (PAIR) {
        // The odd CTA's copies complete on the even CTA's barriers: hand the
        // even CTA this CTA's per-stage copy counts, so that it can drain for
        // both.
        if (!leader && warp == 0 && lane == 0) {
            for (int s = 0; s < CF::STAGES; ++s)
                st_shared_cluster_u32(mapa_shared(smem_addr(const_cast<uint32_t *>(peer_issue_count + s)), 0),
                                      issue_count[s]);
        }
        cluster_sync();
    }
    if (leader && warp == 0 && lane == 0 && *abort_flag) {
        // Some role gave up: copies no one consumed may still be landing.
        // Stage s's copies before the last phase anyone issued were all
        // consumed (a copy is issued only after its slot's previous contents
        // were), so only that last phase can be pending.  With a pair, that
        // phase may have been issued by one CTA only; the even CTA then
        // completes the half that will never come (the odd CTA's bytes, or its
        // own arrival with the odd CTA's byte count) and waits for the half
        // that is in flight.
        for (int s = 0; s < CF::STAGES; ++s) {
            const uint32_t mine = issue_count[s];
            const uint32_t peer = PAIR ? peer_issue_count[s] : mine;
            const uint32_t n = mine > peer ? mine : peer;
            if (n == 0)
                continue;
            if (mine + 1 < n || peer + 1 < n) {
                atomicOr(&g_device_error, ERR_DRAIN);  // cannot happen: the counts differ by one at most
                continue;
            }
            if constexpr (PAIR) {
                if (mine == n && peer + 1 == n)
                    mbar_complete_tx(full_bar(s), CF::STAGE_BYTES);
                else if (peer == n && mine + 1 == n)
                    mbar_arrive_expect_tx(full_bar(s), CF::STAGE_BYTES);
            }
            wait_drain(full_bar(s), (n - 1) & 1u, timeout);
        }
    }
    if constexpr (PAIR)
        cluster_sync();  // the even CTA's MMAs write this CTA's TMEM and read its shared memory
    else
        __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) {
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem_base, CF::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, CF::TMEM_COLS);
    }
}

// Zero-padded copy of a rows x cols matrix of 16-bit values (any alignment of
// `src`) into dst with a row length of dst_cols (a multiple of 8) and a
// 16-byte-aligned base: each thread writes 8 values (16 bytes) at a time,
// read as four 4-byte words when every source word is 4-byte aligned (an even
// row length and a 4-byte-aligned base), else as eight 2-byte values.
// Measured on B200 (the 4000 x 2050 bf16 A of the ragged shape): the 4-byte
// loads and 32-bit index arithmetic take 2.5% off the whole call; one warp per
// row (fewer loads in flight) and copies built from aligned 16-byte source
// words with lane shuffles were slower.
__global__ void __launch_bounds__(256) pad_copy_kernel(const uint16_t *__restrict__ src, int64_t rows,
                                                       int64_t cols, uint16_t *__restrict__ dst,
                                                       int64_t dst_cols)
{
    // launched as a programmatic dependent: src may be the previous kernel's
    // output and dst may still be read by it, so wait for that kernel first;
    // the GEMM that reads dst waits for this kernel in turn
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t chunks_per_row = dst_cols >> 3;
    const int64_t total = rows * chunks_per_row;
    const bool w4 = (reinterpret_cast<uintptr_t>(src) & 3) == 0 && (cols & 1) == 0;
    const bool small = total <= 0x7fffffff;  // 32-bit index arithmetic
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t r, c0;
        if (small) {
            const uint32_t i32 = static_cast<uint32_t>(idx), cpr = static_cast<uint32_t>(chunks_per_row);
            const uint32_t r32 = i32 / cpr;
            r = r32;
            c0 = static_cast<int64_t>(i32 - r32 * cpr) << 3;
        } else {
            r = idx / chunks_per_row;
            c0 = (idx - r * chunks_per_row) << 3;
        }
        const uint16_t *s = src + r * cols;
        uint4 w;
        if (w4) {
            const uint32_t *s32 = reinterpret_cast<const uint32_t *>(s + c0);
            w.x = c0 < cols ? __ldg(s32) : 0u;
            w.y = c0 + 2 < cols ? __ldg(s32 + 1) : 0u;
            w.z = c0 + 4 < cols ? __ldg(s32 + 2) : 0u;
            w.w = c0 + 6 < cols ? __ldg(s32 + 3) : 0u;
        } else {
            uint16_t e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                e[i] = (c0 + i < cols) ? s[c0 + i] : static_cast<uint16_t>(0);
            w.x = e[0] | (static_cast<uint32_t>(e[1]) << 16);
            w.y = e[2] | (static_cast<uint32_t>(e[3]) << 16);
            w.z = e[4] | (static_cast<uint32_t>(e[5]) << 16);
            w.w = e[6] | (static_cast<uint32_t>(e[7]) << 16);
        }
        *reinterpret_cast<uint4 *>(dst + r * dst_cols + c0) = w;
    }
}

} // namespace tl
