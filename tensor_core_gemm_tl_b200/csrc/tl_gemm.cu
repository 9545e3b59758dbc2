// tl_gemm.cu -- host side of libtlgemm.so: for the GEMM, argument
// validation, the launch plan (kernel configuration, padding, store path),
// tensor-map encoding and the launches; the same for the attention forward,
// the row softmax and the vector add; the device error word's read-out.  The
// C ABI is declared in include/tl_gemm.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <random>
#include <unordered_map>

#include "tl_gemm.h"
#include "gemm_kernel.cuh"
#include "attention_kernel.cuh"
#include "rowwise_kernels.cuh"

namespace tl {
namespace {

constexpr uint64_t kDefaultTimeoutNs = 10ull * 1000 * 1000 * 1000;
constexpr int kDefaultRasterGroup = 8;  // output-tile rows per rasterisation group

using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);

struct ConfigEntry {
    const char *name;
    int bm, bn, bk, stages;  // bm: output rows per tile (256 for a CTA pair)
    int cta_m;               // rows of A each CTA loads per tile (the A box height)
    int ctas;                // 1, or 2 for a CTA pair (cluster of two, cta_group::2 MMA)
    int threads;             // threads per CTA
    int smem_bytes;
    KernelFn fn[2][2][3][2];  // [dtype][fused epilogue][store mode][B given transposed]
};

template <class CF, int DT, int EPI, int STORE>
void fill_entry(ConfigEntry &e)
{
    e.fn[DT][EPI][STORE][0] = gemm_sm100_kernel<CF, DT, EPI, STORE, false>;
    e.fn[DT][EPI][STORE][1] = gemm_sm100_kernel<CF, DT, EPI, STORE, true>;
}

template <class CF, int DT, int EPI>
void fill_entry_stores(ConfigEntry &e)
{
    fill_entry<CF, DT, EPI, STORE_ELEMENTS>(e);
    fill_entry<CF, DT, EPI, STORE_TMA>(e);
    fill_entry<CF, DT, EPI, STORE_F32>(e);
}

template <class CF>
ConfigEntry make_entry(const char *name)
{
    ConfigEntry e;
    e.name = name;
    e.bm = CF::TILE_M;
    e.cta_m = CF::BM;
    e.bn = CF::BN;
    e.ctas = CF::CTAS;
    e.threads = CF::THREADS;
    e.bk = CF::BK;
    e.stages = CF::STAGES;
    e.smem_bytes = CF::SMEM_BYTES;
    fill_entry_stores<CF, 0, 0>(e);
    fill_entry_stores<CF, 0, 1>(e);
    fill_entry_stores<CF, 1, 0>(e);
    fill_entry_stores<CF, 1, 1>(e);
    return e;
}

const ConfigEntry &config(int i);
int num_configs();

const ConfigEntry kConfigs[] = {
    make_entry<TileConfig<256, 4>>("bm128_bn256_bk64_s4"),
    make_entry<TileConfig<128, 6>>("bm128_bn128_bk64_s6"),
    make_entry<TileConfig<64, 8>>("bm128_bn64_bk64_s8"),
    make_entry<TileConfig<256, 6, true>>("bm256_bn256_bk64_s6_pair"),
    make_entry<TileConfig<128, 8, true>>("bm256_bn128_bk64_s8_pair"),
};

int num_configs() { return static_cast<int>(sizeof(kConfigs) / sizeof(kConfigs[0])); }
const ConfigEntry &config(int i) { return kConfigs[i]; }

// Shapes measured by the offline sweep: (M, N, K, dtype, epilogue) -> config.
struct TableRow {
    int64_t m, n, k;
    int dtype, epi;
    const char *config;
    int split;  // 1: split the tiles of a short last round; 0: never
    int group;  // output-tile rows per rasterisation group (0: the default)
};
const TableRow kTable[] = {
#include "config_table.inc"
};

int config_index(const char *name)
{
    for (int i = 0; i < num_configs(); ++i)
        if (std::strcmp(kConfigs[i].name, name) == 0)
            return i;
    return -1;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// How the tiles of one launch are cut into work items.  Tiles fill whole
// rounds of `units` (CTAs, or CTA pairs) first.  The tiles of a last, partial
// round would leave units idle for a whole tile's time; instead their
// k-blocks can be spread evenly over up to two units per tile, each unit
// taking one consecutive range (which may end inside the next tile).  A tile
// whose k-blocks fall to several units is summed by the last of them to
// finish (see the kernel): nobody waits, so nothing depends on all units
// being resident.
//
// The split costs the last arrival of each tile a chain of round trips to L2
// (its partial sums out, its arrival count, then every part's sums back in,
// 16 loads in flight each) -- about two k-blocks of a 256-column tile's time
// each, four of a narrower tile's.  Under SPLIT_POLICY the split is taken only
// when the k-blocks it saves exceed that; SPLIT_FORCE takes it whenever the
// last round is partial and every unit gets at least 4 k-blocks.
enum SplitMode { SPLIT_NEVER = 0, SPLIT_POLICY = 1, SPLIT_FORCE = 2 };

struct TailSplit {
    int64_t full_tiles, tail_tiles, tail_units;
    int32_t max_parts;  // most units sharing one tile (1: none shared)
};

TailSplit tail_split(int64_t tiles, int64_t units, int64_t num_kb, int block_n, int mode)
{
    TailSplit t{tiles, 0, 0, 1};
    const int64_t rem = tiles % units;
    if (mode == SPLIT_NEVER || rem == 0 || num_kb < 8)
        return t;
    const int64_t T = rem * num_kb;
    int64_t tail_units = units < 2 * rem ? units : 2 * rem;
    if (tail_units > T / 4)
        tail_units = T / 4;
    if (tail_units <= rem)
        return t;
    // units meeting tail tile r: ceil((x + 1) U / T) - 1 for its first and last k-block x
    int32_t max_parts = 1;
    for (int64_t r = 0; r < rem; ++r) {
        const int64_t first = ((r * num_kb + 1) * tail_units + T - 1) / T - 1;
        const int64_t last = (((r + 1) * num_kb) * tail_units + T - 1) / T - 1;
        if (last - first + 1 > max_parts)
            max_parts = static_cast<int32_t>(last - first + 1);
    }
    if (mode == SPLIT_POLICY) {
        const int64_t saved = num_kb - (T + tail_units - 1) / tail_units;
        const int64_t chunks_per_warp = block_n >= 256 ? 2 : 1;
        const int64_t round_trips = 2 + chunks_per_warp * max_parts;
        const int64_t need = round_trips * (block_n >= 256 ? 2 : 4);
        if (saved < need)
            return t;
    }
    t.full_tiles = tiles - rem;
    t.tail_tiles = rem;
    t.tail_units = tail_units;
    t.max_parts = max_parts;
    return t;
}

// Model for shapes the sweep has not measured: the busiest unit's time, in
// tiles of each configuration weighted by its measured relative tensor-pipe
// efficiency (narrower tiles pull more operand bytes per MMA flop into each
// SM).  Whole rounds of tiles count fully; a split last round counts as the
// k-blocks each unit then takes plus two k-blocks for the partial sums; a
// partial round that is not split counts as a whole one.
int model_config(int64_t M, int64_t N, int64_t K, int num_sms)
{
    // bm128_bn256, bm128_bn128, bm128_bn64, pair 256 x 256, pair 256 x 128
    static const double eff[] = {0.86, 0.67, 0.36, 0.95, 0.68};
    int best = 0;
    double best_cost = 1e300;
    for (int i = 0; i < num_configs(); ++i) {
        const ConfigEntry &c = kConfigs[i];
        const int64_t tiles = ceil_div(M, c.bm) * ceil_div(N, c.bn);
        const int64_t units = num_sms / c.ctas;
        const int64_t num_kb = ceil_div(K, c.bk);
        const TailSplit ts = tail_split(tiles, units, num_kb, c.bn, SPLIT_POLICY);
        double rounds = static_cast<double>(ts.full_tiles / units);
        if (ts.tail_tiles > 0)
            rounds += (static_cast<double>(ceil_div(ts.tail_tiles * num_kb, ts.tail_units)) + 2.0) / num_kb;
        else if (tiles % units)
            rounds += 1.0;
        const double cost = rounds * (static_cast<double>(c.bm) * c.bn / c.ctas) / eff[i];
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = i;
        }
    }
    return best;
}

// The measured choice for this shape (configuration, and whether its last
// round may be cut along K), else the wave model with the split rule of
// tail_split.
int choose_config(int64_t M, int64_t N, int64_t K, int dtype, int epi, int num_sms, int *split_mode, int *group)
{
    for (const TableRow &r : kTable) {
        if (r.m == M && r.n == N && r.k == K && r.dtype == dtype && r.epi == (epi != 0 ? 1 : 0)) {
            const int i = config_index(r.config);
            if (i >= 0) {
                *split_mode = r.split != 0 ? SPLIT_FORCE : SPLIT_NEVER;  // measured: split or not
                *group = r.group;
                return i;
            }
        }
    }
    *split_mode = SPLIT_POLICY;
    *group = 0;
    return model_config(M, N, K, num_sms);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Plan {
    tl_plan pub;
    int64_t lda, ldb;        // row lengths (elements) of the operands the kernel reads
    int64_t a_ws_off, b_ws_off;
    int64_t partial_off, arrival_off;  // split-tile partial sums and their arrival words
    int32_t num_kb;
    int32_t tail_tiles, tail_units, num_slots;
};

bool epi_has_bias(int epi)
{
    return epi == TL_EPI_BIAS_GELU || epi == TL_EPI_BIAS || epi == TL_EPI_BIAS_GELU_TANH;
}

// GELU form of an epilogue: 0 none, 1 exact (erf), 2 tanh
int epi_gelu_form(int epi)
{
    if (epi == TL_EPI_BIAS_GELU || epi == TL_EPI_GELU)
        return 1;
    if (epi == TL_EPI_BIAS_GELU_TANH || epi == TL_EPI_GELU_TANH)
        return 2;
    return 0;
}

// Store mode of the kernel for this call (see StoreMode)
int store_mode(const tl_plan &q, const tl_gemm_options *opt)
{
    if (opt && opt->c_float32)
        return STORE_F32;
    return q.direct_store ? STORE_ELEMENTS : STORE_TMA;
}

tl_status validate(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N,
                   int64_t K, int dtype, int epi, const tl_gemm_options *opt)
{
    if (!A || !B || !C)
        return TL_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0)
        return TL_ERR_INVALID_ARG;
    if (dtype != TL_F16 && dtype != TL_BF16)
        return TL_ERR_INVALID_ARG;
    if (epi < TL_EPI_NONE || epi > TL_EPI_GELU_TANH)
        return TL_ERR_INVALID_ARG;
    const bool needs_bias = epi_has_bias(epi);
    if (needs_bias && !bias)
        return TL_ERR_INVALID_ARG;
    if (opt && (opt->config < 0 || opt->config > num_configs()))
        return TL_ERR_INVALID_ARG;
    if (opt && (opt->inject_fault < 0 || opt->inject_fault > 2))
        return TL_ERR_INVALID_ARG;
    if (opt && ((opt->no_split != 0 && opt->no_split != 1) || (opt->b_layout != 0 && opt->b_layout != 1) ||
                (opt->c_float32 != 0 && opt->c_float32 != 1) || opt->raster_group < 0 ||
                (opt->force_split != 0 && opt->force_split != 1) || (opt->force_split && opt->no_split)))
        return TL_ERR_INVALID_ARG;
    const int64_t lim = 0x7FFFFFFFll;
    if (M > lim || N > lim || K > lim)
        return TL_ERR_UNSUPPORTED;
    const bool c_f32 = opt && opt->c_float32;
    if (!aligned(A, 2) || !aligned(B, 2) || !aligned(C, c_f32 ? 4 : 2) || (needs_bias && !aligned(bias, 2)))
        return TL_ERR_MISALIGNED;
    return TL_OK;
}

tl_status make_plan(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N,
                    int64_t K, int dtype, int epi, int num_sms, int max_units, const tl_gemm_options *opt,
                    Plan *out)
{
    tl_status st = validate(A, B, bias, C, M, N, K, dtype, epi, opt);
    if (st != TL_OK)
        return st;
    if (num_sms <= 0)
        return TL_ERR_INVALID_ARG;
    int split_mode = SPLIT_POLICY;  // a forced configuration follows the cost rule
    int table_group = 0;
    int ci = (opt && opt->config > 0) ? opt->config - 1
                                      : choose_config(M, N, K, dtype, epi, num_sms, &split_mode, &table_group);
    if (opt && opt->no_split)
        split_mode = SPLIT_NEVER;
    else if (opt && opt->force_split)
        split_mode = SPLIT_FORCE;
    const ConfigEntry &c = kConfigs[ci];
    Plan p{};
    tl_plan &q = p.pub;
    q.config = ci;
    q.block_m = c.bm;
    q.block_n = c.bn;
    q.block_k = c.bk;
    q.stages = c.stages;
    q.tiles_m = static_cast<int32_t>(ceil_div(M, c.bm));
    q.tiles_n = static_cast<int32_t>(ceil_div(N, c.bn));
    const int64_t tiles = static_cast<int64_t>(q.tiles_m) * q.tiles_n;
    if (tiles > 0x7FFFFFFFll)
        return TL_ERR_UNSUPPORTED;
    int64_t units = num_sms / c.ctas;
    if (max_units > 0 && max_units < units)
        units = max_units;
    p.num_kb = static_cast<int32_t>(ceil_div(K, c.bk));
    const TailSplit ts = tail_split(tiles, units, p.num_kb, c.bn, split_mode);
    q.split = ts.max_parts;
    q.full_tiles = static_cast<int32_t>(ts.full_tiles);
    p.tail_tiles = static_cast<int32_t>(ts.tail_tiles);
    p.tail_units = static_cast<int32_t>(ts.tail_units);
    p.num_slots = ts.tail_tiles > 0 ? static_cast<int32_t>(ts.tail_units + ts.tail_tiles - 1) : 0;
    q.tail_units = p.tail_units;
    q.num_slots = p.num_slots;
    // units that get work: those with whole tiles, and those with a piece of
    // the split last round
    int64_t busy = ts.full_tiles < units ? ts.full_tiles : units;
    if (ts.tail_tiles > 0 && ts.tail_units > busy)
        busy = ts.tail_units;
    if (ts.tail_tiles == 0)
        busy = tiles < units ? tiles : units;
    q.grid = static_cast<int32_t>(busy * c.ctas);
    q.cluster_ctas = c.ctas;
    q.smem_bytes = c.smem_bytes;
    // TMA needs a 16-byte-aligned base and row strides that are multiples of 16 bytes.
    const bool bt = opt && opt->b_layout == 1;  // B given as N x K
    const int64_t b_cols = bt ? K : N;         // row length of B as stored
    const int64_t b_rows = bt ? N : K;
    q.pad_a = !(aligned(A, 16) && K % 8 == 0);
    q.pad_b = !(aligned(B, 16) && b_cols % 8 == 0);
    q.direct_store = (opt && opt->c_float32) || !(aligned(C, 16) && N % 8 == 0);
    // A padded copy gets rows of a whole number of 128-byte lines (64
    // elements): every 64-element box row of the tiled loads is then one
    // line, not two.  Measured on 4000 x 3000 x 2056 bf16, where B's rows
    // (6000 bytes) are unaligned too, lines shared between box rows cost 15%
    // of the GEMM's time.
    p.lda = q.pad_a ? ceil_div(K, 64) * 64 : K;
    p.ldb = q.pad_b ? ceil_div(b_cols, 64) * 64 : b_cols;
    int64_t ws = 0;
    p.a_ws_off = p.b_ws_off = -1;
    if (q.pad_a) {
        p.a_ws_off = ws;
        ws += ceil_div(M * p.lda * 2, 256) * 256;
    }
    if (q.pad_b) {
        p.b_ws_off = ws;
        ws += ceil_div(b_rows * p.ldb * 2, 256) * 256;
    }
    p.partial_off = p.arrival_off = -1;
    if (ts.tail_tiles > 0) {
        // one 128 x BN fp32 slab per (slot, CTA of the pair); one arrival word
        // per (tail tile, CTA, TMEM lane quarter, epilogue warp of the quarter)
        const int64_t slabs = static_cast<int64_t>(p.num_slots) * c.ctas;
        p.partial_off = ws;
        ws += ceil_div(slabs * 128 * c.bn * 4, 256) * 256;
        p.arrival_off = ws;
        ws += ceil_div(ts.tail_tiles * c.ctas * 4 * 2 * 8, 256) * 256;
    }
    q.workspace_bytes = ws;
    int group = (opt && opt->raster_group > 0) ? opt->raster_group : (table_group > 0 ? table_group : kDefaultRasterGroup);
    if (group > q.tiles_m)
        group = q.tiles_m;
    q.raster_group = group;
    *out = p;
    return TL_OK;
}

// ------------------------------------------------------------------ driver API
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D row-major matrix of 16-bit values: `rows` x `cols`, row length `ld`;
// box of box_cols (<= 64, 128 B) x box_rows, 128-byte swizzle.
bool encode_2d(CUtensorMap *map, const void *base, int dtype, int64_t rows, int64_t cols, int64_t ld,
               int box_cols, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = dtype == TL_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ per-device state
struct DeviceState {
    int num_sms = 0;
    int cc_major = 0;
    cudaMemPool_t pool = nullptr;
    std::unordered_map<const void *, bool> smem_set;  // kernels whose smem limit is raised
    std::unordered_map<const void *, int> max_clusters;  // resident clusters of two, per kernel
};

std::mutex g_mu;
std::unordered_map<int, DeviceState> g_dev;

tl_status device_state(DeviceState **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return TL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState &d = g_dev[dev];
    if (d.num_sms == 0) {
        int sms = 0, major = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return TL_ERR_CUDA;
        d.num_sms = sms;
        d.cc_major = major;
    }
    *out = &d;
    return TL_OK;
}

tl_status ensure_pool(DeviceState *d)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (d->pool)
        return TL_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return TL_ERR_CUDA;
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    if (cudaMemPoolCreate(&d->pool, &props) != cudaSuccess)
        return TL_ERR_CUDA;
    uint64_t keep = ~0ull;  // keep freed blocks for reuse by later calls
    cudaMemPoolSetAttribute(d->pool, cudaMemPoolAttrReleaseThreshold, &keep);
    return TL_OK;
}

tl_status raise_smem_limit(DeviceState *d, KernelFn fn, int bytes)
{
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = d->smem_set.find(reinterpret_cast<const void *>(fn));
    if (it != d->smem_set.end())
        return TL_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return TL_ERR_CUDA;
    d->smem_set[reinterpret_cast<const void *>(fn)] = true;
    return TL_OK;
}

tl_status max_active_clusters(DeviceState *d, KernelFn fn, const cudaLaunchConfig_t &cfg, int *out)
{
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = d->max_clusters.find(reinterpret_cast<const void *>(fn));
        if (it != d->max_clusters.end()) {
            *out = it->second;
            return TL_OK;
        }
    }
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess)
        return TL_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    d->max_clusters[reinterpret_cast<const void *>(fn)] = n;
    *out = n;
    return TL_OK;
}

tl_status launch_pad(const void *src, int64_t rows, int64_t cols, void *dst, int64_t dst_cols, int num_sms,
                     cudaStream_t stream)
{
    const int64_t work = rows * (dst_cols / 8);  // 16-byte destination words
    int64_t blocks = ceil_div(work, 256);
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    // a programmatic dependent launch, like the GEMM's: the copy's launch
    // overlaps the end of the previous kernel on the stream
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, pad_copy_kernel, static_cast<const uint16_t *>(src), rows,
                                               cols, static_cast<uint16_t *>(dst), dst_cols);
    return err == cudaSuccess && cudaGetLastError() == cudaSuccess ? TL_OK : TL_ERR_CUDA;
}

// Launch the GEMM itself with operands the kernel can read through TMA.
std::atomic<unsigned long long> g_epoch{0};

// A launch stamp below 2^56 (it shares a 64-bit arrival word with an 8-bit
// count) that no earlier launch of this process has used, starting from a
// random point so that memory left by another process never matches it.
unsigned long long next_epoch()
{
    constexpr unsigned long long kMask = (1ull << 56) - 1;
    unsigned long long e = g_epoch.fetch_add(1) + 1;
    if (e == 1) {
        std::random_device rd;
        const unsigned long long base = (((static_cast<unsigned long long>(rd()) << 32) ^ rd()) & kMask) | 1ull;
        unsigned long long expected = 1;
        g_epoch.compare_exchange_strong(expected, base);
        e = g_epoch.fetch_add(1) + 1;
    }
    e &= kMask;
    return e ? e : 1ull;
}

tl_status launch_gemm(const Plan &p, const void *A, const void *B, const void *bias, void *C, int64_t M,
                      int64_t N, int64_t K, int dtype, int epi, cudaStream_t stream, DeviceState *d,
                      const tl_gemm_options *opt, void *workspace)
{
    const ConfigEntry &c = kConfigs[p.pub.config];
    const int store = store_mode(p.pub, opt);
    const bool tma_store = store == STORE_TMA;
    const int bt = (opt && opt->b_layout == 1) ? 1 : 0;
    KernelFn fn = c.fn[dtype][epi != 0][store][bt];
    tl_status st = raise_smem_limit(d, fn, c.smem_bytes);
    if (st != TL_OK)
        return st;

    CUtensorMap ta, tb, tc;
    std::memset(&tc, 0, sizeof(tc));
    // test hook 2: the driver "refuses" A's tensor map, as a failing encode would
    const bool refuse_encode = opt && opt->inject_fault == 2;
    if (refuse_encode || !encode_2d(&ta, A, dtype, M, K, p.lda, 64, c.cta_m))
        return TL_ERR_CUDA;
    if (bt ? !encode_2d(&tb, B, dtype, N, K, p.ldb, 64, c.bn / c.ctas)   // B^T: BN/CTAS rows of 64 k
           : !encode_2d(&tb, B, dtype, K, N, p.ldb, 64, c.bk))
        return TL_ERR_CUDA;
    if (tma_store && !encode_2d(&tc, C, dtype, M, N, N, 64, 32))
        return TL_ERR_CUDA;

    GemmParams gp{};
    gp.M = static_cast<int32_t>(M);
    gp.N = static_cast<int32_t>(N);
    gp.K = static_cast<int32_t>(K);
    gp.tiles_m = p.pub.tiles_m;
    gp.tiles_n = p.pub.tiles_n;
    gp.num_tiles = p.pub.tiles_m * p.pub.tiles_n;
    gp.num_kb = static_cast<int32_t>(ceil_div(K, c.bk));
    gp.group_m = p.pub.raster_group;
    gp.bias = static_cast<const uint16_t *>(bias);
    gp.bias_vec16 = bias && aligned(bias, 16);
    gp.epi_bias = epi_has_bias(epi);
    gp.epi_gelu = epi_gelu_form(epi);
    if (!gp.epi_bias)
        gp.bias = nullptr;
    gp.inject_fault = (opt && opt->inject_fault == 1) ? 1 : 0;
    gp.C = static_cast<uint16_t *>(C);
    gp.C32 = store == STORE_F32 ? static_cast<float *>(C) : nullptr;
    gp.c32_vec16 = store == STORE_F32 && aligned(C, 16) && N % 4 == 0;
    gp.ldc = N;
    gp.timeout_ns = (opt && opt->timeout_ns) ? opt->timeout_ns : kDefaultTimeoutNs;
    gp.full_tiles = p.pub.full_tiles;
    gp.tail_tiles = p.tail_tiles;
    gp.tail_units = p.tail_units;
    gp.num_slots = p.num_slots;
    gp.partials = nullptr;
    gp.arrivals = nullptr;
    gp.epoch = 0;
    if (p.tail_tiles > 0) {
        if (!workspace)
            return TL_ERR_INVALID_ARG;
        gp.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + p.partial_off);
        gp.arrivals = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + p.arrival_off);
        gp.epoch = next_epoch();
    }

    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    cfg.gridDim = dim3(static_cast<unsigned>(p.pub.grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(c.threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(c.smem_bytes);
    cfg.stream = stream;
    // The kernel's set-up may overlap the previous kernel on the stream: it
    // waits for that kernel (griddepcontrol.wait) before touching global memory.
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (c.ctas == 2) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 2;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    if (cudaLaunchKernelEx(&cfg, fn, ta, tb, tc, gp) != cudaSuccess)
        return TL_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ERR_CUDA;
}

// The plan for this device: for CTA-pair configurations, no more pairs than
// can be resident at once (a persistent unit that is not resident would only
// start when another has finished all its work).
tl_status device_plan(DeviceState *d, const void *A, const void *B, const void *bias, void *C, int64_t M,
                      int64_t N, int64_t K, int dtype, int epi, const tl_gemm_options *opt, Plan *p)
{
    tl_status st = make_plan(A, B, bias, C, M, N, K, dtype, epi, d->num_sms, 0, opt, p);
    if (st != TL_OK)
        return st;
    const ConfigEntry &c = kConfigs[p->pub.config];
    if (c.ctas != 2)
        return TL_OK;
    KernelFn fn = c.fn[dtype][epi != 0][store_mode(p->pub, opt)][(opt && opt->b_layout == 1) ? 1 : 0];
    if ((st = raise_smem_limit(d, fn, c.smem_bytes)) != TL_OK)
        return st;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(c.threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(c.smem_bytes);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int max_clusters = 0;
    if ((st = max_active_clusters(d, fn, cfg, &max_clusters)) != TL_OK)
        return st;
    if (max_clusters <= 0)
        return TL_ERR_CUDA;
    if (max_clusters < d->num_sms / 2)
        st = make_plan(A, B, bias, C, M, N, K, dtype, epi, d->num_sms, max_clusters, opt, p);
    return st;
}

tl_status gemm_impl(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N, int64_t K,
                    int dtype, int epi, cudaStream_t stream, const tl_gemm_options *opt)
{
    tl_status st = validate(A, B, bias, C, M, N, K, dtype, epi, opt);
    if (st != TL_OK)
        return st;
    DeviceState *d = nullptr;
    if ((st = device_state(&d)) != TL_OK)
        return st;
    if (d->cc_major != 10)
        return TL_ERR_UNSUPPORTED;
    Plan p;
    if ((st = device_plan(d, A, B, bias, C, M, N, K, dtype, epi, opt, &p)) != TL_OK)
        return st;

    if (p.pub.workspace_bytes == 0)
        return launch_gemm(p, A, B, bias, C, M, N, K, dtype, epi, stream, d, opt, nullptr);

    if ((st = ensure_pool(d)) != TL_OK)
        return st;
    void *ws = nullptr;
    if (cudaMallocFromPoolAsync(&ws, static_cast<size_t>(p.pub.workspace_bytes), d->pool, stream) != cudaSuccess)
        return TL_ERR_CUDA;
    const void *a_use = A, *b_use = B;
    if (p.pub.pad_a) {
        void *dst = static_cast<uint8_t *>(ws) + p.a_ws_off;
        st = launch_pad(A, M, K, dst, p.lda, d->num_sms, stream);
        a_use = dst;
    }
    if (st == TL_OK && p.pub.pad_b) {
        void *dst = static_cast<uint8_t *>(ws) + p.b_ws_off;
        const bool bt = opt && opt->b_layout == 1;
        st = launch_pad(B, bt ? N : K, bt ? K : N, dst, p.ldb, d->num_sms, stream);
        b_use = dst;
    }
    if (st == TL_OK)
        st = launch_gemm(p, a_use, b_use, bias, C, M, N, K, dtype, epi, stream, d, opt, ws);
    if (cudaFreeAsync(ws, stream) != cudaSuccess && st == TL_OK)
        st = TL_ERR_CUDA;
    return st;
}

// ------------------------------------------------------------------ attention forward
using AttnFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, AttnParams);

struct AttnEntry {
    int smem_bytes;
    int threads;
    int launch_regs;     // registers a thread the warpgroup register split needs at launch
    int tiles_per_cta;   // 128-row query tiles one CTA computes
    AttnFn fn[2];        // [dtype]
};

// Two query tiles per CTA in ping-pong (attention_kernel.cuh)
template <int D>
AttnEntry make_attn_entry()
{
    using CF = AttnConfig<D>;
    AttnEntry e;
    e.smem_bytes = CF::SMEM_BYTES;
    e.threads = CF::THREADS;
    e.launch_regs = CF::LAUNCH_REGS;
    e.tiles_per_cta = CF::TILES;
    e.fn[0] = attention_fwd_kernel<CF, 0>;
    e.fn[1] = attention_fwd_kernel<CF, 1>;
    return e;
}

const AttnEntry kAttn64 = make_attn_entry<64>();
const AttnEntry kAttn128 = make_attn_entry<128>();

// [BH][S][D] 16-bit tensor as a 3-D map (D innermost), box 64 x 128 x 1,
// 128-byte swizzle: rows past S read as zero within each (batch, head).
bool encode_3d_rows(CUtensorMap *map, const void *base, int dtype, int64_t BH, int64_t S, int64_t D)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S * D) * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = dtype == TL_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return fn(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

tl_status attention_validate(const void *Q, const void *K, const void *V, void *O, const float *lse, int64_t batch,
                             int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim, int dtype, int causal,
                             float softmax_scale)
{
    if (!Q || !K || !V || !O)
        return TL_ERR_INVALID_ARG;
    if (batch < 1 || heads < 1 || seq_q < 1 || seq_k < 1)
        return TL_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128)
        return TL_ERR_UNSUPPORTED;
    if (dtype != TL_F16 && dtype != TL_BF16)
        return TL_ERR_INVALID_ARG;
    if (!(softmax_scale >= 0.0f) || softmax_scale == INFINITY)
        return TL_ERR_INVALID_ARG;
    // the grid is (pairs of 128-row query tiles, batch * heads), transposed when causal
    const int64_t grid_y = causal ? ceil_div(seq_q, 256) : batch * heads;
    const int64_t grid_x = causal ? batch * heads : ceil_div(seq_q, 256);
    if (grid_y > 65535 || grid_x > 0x7FFFFFFFll || batch * heads > 0x7FFFFFFFll || seq_k > 0x7FFFFFFFll)
        return TL_ERR_UNSUPPORTED;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || (lse && !aligned(lse, 4)))
        return TL_ERR_MISALIGNED;
    return TL_OK;
}

tl_status attention_impl(const void *Q, const void *K, const void *V, void *O, float *lse, int64_t batch,
                         int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim, int dtype, int causal,
                         float softmax_scale, cudaStream_t stream)
{
    tl_status st =
        attention_validate(Q, K, V, O, lse, batch, heads, seq_q, seq_k, head_dim, dtype, causal, softmax_scale);
    if (st != TL_OK)
        return st;
    DeviceState *d = nullptr;
    if ((st = device_state(&d)) != TL_OK)
        return st;
    if (d->cc_major != 10)
        return TL_ERR_UNSUPPORTED;
    const AttnEntry &e = head_dim == 64 ? kAttn64 : kAttn128;
    AttnFn fn = e.fn[dtype];
    {
        // the kernel moves registers between warpgroups; that only fits if
        // it is launched with at least launch_regs a thread
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess)
            return TL_ERR_CUDA;
        if (fa.numRegs < e.launch_regs)
            return TL_ERR_UNSUPPORTED;
    }
    if ((st = raise_smem_limit(d, reinterpret_cast<KernelFn>(fn), e.smem_bytes)) != TL_OK)
        return st;
    const int64_t BH = batch * heads;
    CUtensorMap tq, tk, tv;
    if (!encode_3d_rows(&tq, Q, dtype, BH, seq_q, head_dim) || !encode_3d_rows(&tk, K, dtype, BH, seq_k, head_dim) ||
        !encode_3d_rows(&tv, V, dtype, BH, seq_k, head_dim))
        return TL_ERR_CUDA;
    AttnParams ap{};
    ap.Sq = static_cast<int32_t>(seq_q);
    ap.Sk = static_cast<int32_t>(seq_k);
    ap.BH = static_cast<int32_t>(BH);
    ap.num_qtiles = static_cast<int32_t>(ceil_div(seq_q, 128));
    ap.causal = causal ? 1 : 0;
    const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(head_dim));
    ap.scale_log2 = scale * 1.4426950408889634f;
    ap.O = static_cast<uint16_t *>(O);
    ap.lse = lse;
    ap.timeout_ns = kDefaultTimeoutNs;

    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    // blocks start x fastest.  Non-causal: query-tile pairs along x (the CTAs
    // running together share a head's K and V in L2).  Causal: heads along x,
    // pairs along y reversed in the kernel, so every head's heaviest pair
    // starts before any lighter one.
    const unsigned pairs = static_cast<unsigned>(ceil_div(ap.num_qtiles, e.tiles_per_cta));
    cfg.gridDim = causal ? dim3(static_cast<unsigned>(BH), pairs, 1) : dim3(pairs, static_cast<unsigned>(BH), 1);
    cfg.blockDim = dim3(static_cast<unsigned>(e.threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(e.smem_bytes);
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, tq, tk, tv, ap) != cudaSuccess)
        return TL_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ERR_CUDA;
}

// ------------------------------------------------------------------ row softmax and vector add
// Largest dynamic shared memory the row-in-shared-memory softmax takes (one
// row of 16-bit values plus 16 bytes of alignment slack).
constexpr int64_t kSoftmaxSmemMax = 220 * 1024;

// Persistent grid for a row kernel: one CTA per row, at most as many as can
// be resident at once on every SM (so no CTA waits for a second wave).
template <class Fn>
int64_t resident_grid(DeviceState *d, Fn fn, int threads, size_t smem, int64_t work_blocks)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t cap = static_cast<int64_t>(d->num_sms) * per_sm;
    return work_blocks < cap ? work_blocks : cap;
}

tl_status softmax_impl(const void *X, void *Y, int64_t rows, int64_t cols, int dtype, cudaStream_t stream)
{
    if (!X || !Y || rows < 1 || cols < 1)
        return TL_ERR_INVALID_ARG;
    if (dtype != TL_F16 && dtype != TL_BF16)
        return TL_ERR_INVALID_ARG;
    if (cols > 0x7FFFFFFFll)
        return TL_ERR_UNSUPPORTED;
    if (!aligned(X, 2) || !aligned(Y, 2))
        return TL_ERR_MISALIGNED;
    DeviceState *d = nullptr;
    tl_status st = device_state(&d);
    if (st != TL_OK)
        return st;
    const bool vec = cols % 8 == 0 && aligned(X, 16) && aligned(Y, 16);
    const uint16_t *x = static_cast<const uint16_t *>(X);
    uint16_t *y = static_cast<uint16_t *>(Y);
    const int c = static_cast<int>(cols);
    if (cols <= 1024) {
        // lanes per row: short rows share a warp (rows of up to 128 values take
        // 8 lanes, 16 values each)
        const int lpr = cols <= 128 ? 8 : 32;
        const int64_t work = ceil_div(rows, 8 * (32 / lpr));
        const dim3 b(256);
#define TL_SOFTMAX_WARP_LAUNCH(DT, P, V, L)                                                          \
    do {                                                                                             \
        auto fn = softmax_rows_warp_kernel<DT, P, V, L>;                                             \
        const dim3 g(static_cast<unsigned>(resident_grid(d, fn, 256, 0, work)));                     \
        fn<<<g, b, 0, stream>>>(x, y, rows, c);                                                      \
    } while (0)
#define TL_SOFTMAX_WARP(DT, V)                                                                       \
    do {                                                                                             \
        if (cols <= 64)                                                                              \
            TL_SOFTMAX_WARP_LAUNCH(DT, 8, V, 8);                                                     \
        else if (cols <= 128)                                                                        \
            TL_SOFTMAX_WARP_LAUNCH(DT, 16, V, 8);                                                    \
        else if (cols <= 256)                                                                        \
            TL_SOFTMAX_WARP_LAUNCH(DT, 8, V, 32);                                                    \
        else                                                                                         \
            TL_SOFTMAX_WARP_LAUNCH(DT, 32, V, 32);                                                   \
    } while (0)
        if (dtype == TL_BF16) {
            if (vec)
                TL_SOFTMAX_WARP(1, true);
            else
                TL_SOFTMAX_WARP(1, false);
        } else {
            if (vec)
                TL_SOFTMAX_WARP(0, true);
            else
                TL_SOFTMAX_WARP(0, false);
        }
#undef TL_SOFTMAX_WARP
#undef TL_SOFTMAX_WARP_LAUNCH
    } else if (vec && cols <= 16384) {
        // the row in registers: 256 or 512 threads x up to 32 values, one read
        const int threads = cols <= 4096 ? 256 : 512;
        const dim3 b(threads);
        auto launch = [&](auto fn) {
            const dim3 g(static_cast<unsigned>(resident_grid(d, fn, threads, 0, rows)));
            fn<<<g, b, 0, stream>>>(x, y, rows, c);
        };
        if (cols <= 8192)
            dtype == TL_BF16 ? launch(softmax_rows_cta_regs_kernel<1, 16>) : launch(softmax_rows_cta_regs_kernel<0, 16>);
        else
            dtype == TL_BF16 ? launch(softmax_rows_cta_regs_kernel<1, 32>) : launch(softmax_rows_cta_regs_kernel<0, 32>);
    } else if (ceil_div(2 * cols + 16, 128) * 128 + 128 <= kSoftmaxSmemMax) {
        // the row in shared memory, read from HBM once by bulk copies; two
        // row buffers when they fit, so the next row streams in meanwhile
        const int buf_bytes = static_cast<int>(ceil_div(2 * cols + 16, 128) * 128);
        // two CTAs of one row buffer each when both fit on an SM (two rows'
        // reductions overlap), else one CTA with two buffers when they fit
        // (the next row streams in during the reductions), else one buffer
        const bool two_ctas = 2 * (static_cast<int64_t>(buf_bytes) + 128 + 1024) <= kSoftmaxSmemMax;
        const int nbuf = !two_ctas && 2 * static_cast<int64_t>(buf_bytes) + 128 <= kSoftmaxSmemMax ? 2 : 1;
        const int smem = nbuf * buf_bytes + 128;  // + slack to a 128-byte boundary
        const dim3 b(512);
        // y's body takes whole words when y lies as far from a 16-byte
        // boundary as x (then every row's x and y do)
        const int y_vec = ((reinterpret_cast<uintptr_t>(X) - reinterpret_cast<uintptr_t>(Y)) & 15) == 0;
        auto launch = [&](auto fn) -> tl_status {
            tl_status r = raise_smem_limit(d, reinterpret_cast<KernelFn>(fn), static_cast<int>(kSoftmaxSmemMax));
            if (r != TL_OK)
                return r;
            const dim3 g(static_cast<unsigned>(resident_grid(d, fn, 512, static_cast<size_t>(smem), rows)));
            fn<<<g, b, smem, stream>>>(x, y, rows, c, y_vec, nbuf, buf_bytes, kDefaultTimeoutNs);
            return TL_OK;
        };
        if ((st = dtype == TL_BF16 ? launch(softmax_rows_smem_kernel<1>) : launch(softmax_rows_smem_kernel<0>)) != TL_OK)
            return st;
    } else {
        int64_t blocks = rows;
        const int64_t cap = static_cast<int64_t>(d->num_sms) * 4;
        if (blocks > cap)
            blocks = cap;
        const dim3 g(static_cast<unsigned>(blocks)), b(512);
        // vectors in the body of every row when x and y sit equally far from a 16-byte boundary
        const int peel = ((reinterpret_cast<uintptr_t>(X) - reinterpret_cast<uintptr_t>(Y)) & 15) == 0;
        if (dtype == TL_BF16)
            softmax_rows_block_kernel<1><<<g, b, 0, stream>>>(x, y, rows, cols, peel);
        else
            softmax_rows_block_kernel<0><<<g, b, 0, stream>>>(x, y, rows, cols, peel);
    }
    return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ERR_CUDA;
}

tl_status vector_add_impl(const float *A, const float *B, float *C, int64_t n, cudaStream_t stream)
{
    if (!A || !B || !C || n < 1)
        return TL_ERR_INVALID_ARG;
    if (!aligned(A, 4) || !aligned(B, 4) || !aligned(C, 4))
        return TL_ERR_MISALIGNED;
    DeviceState *d = nullptr;
    tl_status st = device_state(&d);
    if (st != TL_OK)
        return st;
    const int vec = aligned(A, 16) && aligned(B, 16) && aligned(C, 16);
    int64_t blocks = ceil_div(vec ? ceil_div(n, 4) : n, 256);
    const int64_t cap = static_cast<int64_t>(d->num_sms) * 16;
    if (blocks > cap)
        blocks = cap;
    vector_add_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(A, B, C, n, vec);
    return cudaGetLastError() == cudaSuccess ? TL_OK : TL_ERR_CUDA;
}

// ------------------------------------------------------------------ allocation-free entry point
// The scratch area of tl_gemm_noalloc: file scope, one per device, reserved
// when the module is loaded.  Host code may only use the address that
// cudaGetSymbolAddress returns for the current device, never the name.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoallocDevices = 64;
std::atomic<void *> g_noalloc_scratch_ptr[kMaxNoallocDevices];

// One-time set-up per device (the device must be current): the scratch area's
// device address, and every kernel's shared-memory limit and cluster
// occupancy, so that later calls touch no allocator and insert into no map.
tl_status noalloc_setup(DeviceState *d, void **scratch)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return TL_ERR_CUDA;
    if (dev < 0 || dev >= kMaxNoallocDevices)
        return TL_ERR_UNSUPPORTED;
    void *p = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p) {
        *scratch = p;
        return TL_OK;
    }
    static std::mutex mu;
    std::lock_guard<std::mutex> lk(mu);
    p = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
            return TL_ERR_CUDA;
        for (int i = 0; i < num_configs(); ++i) {
            const ConfigEntry &c = kConfigs[i];
            for (int dt = 0; dt < 2; ++dt)
                for (int epi = 0; epi < 2; ++epi)
                    for (int st = 0; st < 2; ++st)
                        for (int bt = 0; bt < 2; ++bt) {
                            KernelFn fn = c.fn[dt][epi][st][bt];
                            tl_status r = raise_smem_limit(d, fn, c.smem_bytes);
                            if (r != TL_OK)
                                return r;
                            if (c.ctas == 2) {
                                cudaLaunchConfig_t cfg{};
                                cudaLaunchAttribute attr[1];
                                attr[0].id = cudaLaunchAttributeClusterDimension;
                                attr[0].val.clusterDim.x = 2;
                                attr[0].val.clusterDim.y = 1;
                                attr[0].val.clusterDim.z = 1;
                                cfg.gridDim = dim3(2, 1, 1);
                                cfg.blockDim = dim3(static_cast<unsigned>(c.threads), 1, 1);
                                cfg.dynamicSmemBytes = static_cast<size_t>(c.smem_bytes);
                                cfg.attrs = attr;
                                cfg.numAttrs = 1;
                                int n = 0;
                                if ((r = max_active_clusters(d, fn, cfg, &n)) != TL_OK)
                                    return r;
                            }
                        }
        }
        p = addr;
        g_noalloc_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    *scratch = p;
    return TL_OK;
}

tl_status gemm_noalloc_impl(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N,
                            int64_t K, int dtype, int epi, cudaStream_t stream)
{
    tl_status st = validate(A, B, bias, C, M, N, K, dtype, epi, nullptr);
    if (st != TL_OK)
        return st;
    DeviceState *d = nullptr;
    if ((st = device_state(&d)) != TL_OK)
        return st;
    if (d->cc_major != 10)
        return TL_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((st = noalloc_setup(d, &scratch)) != TL_OK)
        return st;
    Plan p;
    if ((st = device_plan(d, A, B, bias, C, M, N, K, dtype, epi, nullptr, &p)) != TL_OK)
        return st;
    if (p.pub.workspace_bytes == 0)
        return launch_gemm(p, A, B, bias, C, M, N, K, dtype, epi, stream, d, nullptr, nullptr);
    if (static_cast<uint64_t>(p.pub.workspace_bytes) > TL_NOALLOC_SCRATCH_BYTES)
        return TL_ERR_SCRATCH_LIMIT;
    // the padded copies overwrite every byte of scratch that the GEMM reads; the
    // split-tile partials are written before they are read, under flags stamped
    // with this launch's own epoch
    const void *a_use = A, *b_use = B;
    if (p.pub.pad_a) {
        void *dst = static_cast<uint8_t *>(scratch) + p.a_ws_off;
        if ((st = launch_pad(A, M, K, dst, p.lda, d->num_sms, stream)) != TL_OK)
            return st;
        a_use = dst;
    }
    if (p.pub.pad_b) {
        void *dst = static_cast<uint8_t *>(scratch) + p.b_ws_off;
        if ((st = launch_pad(B, K, N, dst, p.ldb, d->num_sms, stream)) != TL_OK)
            return st;
        b_use = dst;
    }
    return launch_gemm(p, a_use, b_use, bias, C, M, N, K, dtype, epi, stream, d, nullptr, scratch);
}

} // namespace
} // namespace tl

extern "C" {

tl_status tl_gemm_noalloc(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N,
                          int64_t K, tl_dtype dtype, tl_epilogue epi, tl_stream stream)
{
    return tl::gemm_noalloc_impl(A, B, bias, C, M, N, K, dtype, epi, static_cast<cudaStream_t>(stream));
}


tl_status tl_gemm(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N, int64_t K,
                  tl_dtype dtype, tl_epilogue epi, tl_stream stream)
{
    return tl::gemm_impl(A, B, bias, C, M, N, K, dtype, epi, static_cast<cudaStream_t>(stream), nullptr);
}

tl_status tl_gemm_ex(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N, int64_t K,
                     tl_dtype dtype, tl_epilogue epi, tl_stream stream, const tl_gemm_options *options)
{
    return tl::gemm_impl(A, B, bias, C, M, N, K, dtype, epi, static_cast<cudaStream_t>(stream), options);
}

tl_status tl_attention_fwd(const void *Q, const void *K, const void *V, void *O, float *lse, int64_t batch,
                           int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim, tl_dtype dtype,
                           int32_t causal, float softmax_scale, tl_stream stream)
{
    return tl::attention_impl(Q, K, V, O, lse, batch, heads, seq_q, seq_k, head_dim, dtype, causal, softmax_scale,
                              static_cast<cudaStream_t>(stream));
}

tl_status tl_softmax_rows(const void *X, void *Y, int64_t rows, int64_t cols, tl_dtype dtype, tl_stream stream)
{
    return tl::softmax_impl(X, Y, rows, cols, dtype, static_cast<cudaStream_t>(stream));
}

tl_status tl_vector_add(const float *A, const float *B, float *C, int64_t n, tl_stream stream)
{
    return tl::vector_add_impl(A, B, C, n, static_cast<cudaStream_t>(stream));
}

tl_status tl_check_device(tl_stream stream, uint32_t *detail)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return TL_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, tl::g_device_error, sizeof(v)) != cudaSuccess)
        return TL_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(tl::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return TL_ERR_CUDA;
    if (detail)
        *detail = v;
    return v ? TL_ERR_DEVICE_TIMEOUT : TL_OK;
}

tl_status tl_gemm_plan(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N, int64_t K,
                       tl_dtype dtype, tl_epilogue epi, int32_t num_sms, const tl_gemm_options *options,
                       tl_plan *plan)
{
    if (!plan)
        return TL_ERR_INVALID_ARG;
    tl_status st = tl::validate(A, B, bias, C, M, N, K, dtype, epi, options);
    if (st != TL_OK)
        return st;
    if (num_sms <= 0) {
        tl::DeviceState *d = nullptr;
        if ((st = tl::device_state(&d)) != TL_OK)
            return st;
        num_sms = d->num_sms;
    }
    tl::Plan p;
    st = tl::make_plan(A, B, bias, C, M, N, K, dtype, epi, num_sms, 0, options, &p);
    if (st == TL_OK)
        *plan = p.pub;
    return st;
}

int32_t tl_num_configs(void) { return tl::num_configs(); }

const char *tl_config_name(int32_t i)
{
    if (i < 0 || i >= tl::num_configs())
        return nullptr;
    return tl::config(i).name;
}

const char *tl_status_string(tl_status s)
{
    switch (s) {
    case TL_OK: return "TL_OK";
    case TL_ERR_INVALID_ARG: return "TL_ERR_INVALID_ARG";
    case TL_ERR_UNSUPPORTED: return "TL_ERR_UNSUPPORTED";
    case TL_ERR_MISALIGNED: return "TL_ERR_MISALIGNED";
    case TL_ERR_CUDA: return "TL_ERR_CUDA";
    case TL_ERR_DEVICE_TIMEOUT: return "TL_ERR_DEVICE_TIMEOUT";
    case TL_ERR_SCRATCH_LIMIT: return "TL_ERR_SCRATCH_LIMIT";
    }
    return "TL_ERR_UNKNOWN";
}

int32_t tl_version(void) { return TL_VERSION; }

} // extern "C"
