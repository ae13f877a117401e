// nvfp4sk.cu -- C ABI of libnvfp4sk (declared in include/nvfp4sk.h): host-side
// argument checks, tensor-map encoding, launch configuration and the device
// status word.  All kernels live in the *.cuh files included below (one
// translation unit, so that the device error word is a single variable).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "attn.cuh"
#include "common.cuh"
#include "glue.cuh"
#include "linear.cuh"
#include "quant.cuh"
#include "restore.cuh"
#include "wide.cuh"

using namespace nvfp4sk;

namespace {

thread_local std::string t_last_error;
int g_opt_pdl = 1;
int64_t g_opt_timeout_ns = 1000000000ll;
int g_opt_attn_splits = 0;
int g_opt_linear_ctas = 0;
int g_opt_attn_fused = 0;

int fail(int code, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(NVFP4SK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DevInfo {
    int sms = 0;
    int major = 0, minor = 0;
    std::atomic<bool> ready{false};   // set (release) after the fields above are filled
};
constexpr int MAX_DEV = 64;
DevInfo g_dev[MAX_DEV];
std::mutex g_mu;

template <typename K> cudaError_t set_smem(K kern, size_t bytes)
{
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}
template <typename K> cudaError_t allow_big_cluster(K kern)
{
    return cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

// Per device: query the SM count, check sm_100, set kernel attributes once.
int device_info(DevInfo **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEV) return fail(NVFP4SK_ERR_DEVICE, "device id %d out of range", dev);
    DevInfo &d = g_dev[dev];
    if (!d.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!d.ready.load(std::memory_order_relaxed)) {
            if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return cuda_fail(e, "cudaDeviceGetAttribute");
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
            if (d.major != 10 || d.minor != 0)
                return fail(NVFP4SK_ERR_DEVICE, "libnvfp4sk is built for sm_100a; device %d is sm_%d%d", dev,
                            d.major, d.minor);
            cudaError_t es[] = {
                set_smem(nvfp4_linear_kernel<false>, LIN_SMEM_BYTES),
                set_smem(nvfp4_linear_kernel<true>, LIN_SMEM_BYTES_SW),
                set_smem(tree_attn_split_kernel, ATT_SMEM_BYTES),
                set_smem(kv_page_restore_kernel, RST_SMEM_BUDGET + 1024),
                set_smem(nvfp4_linear_wide_kernel, WD_SMEM_BYTES),
                allow_big_cluster(quant_fused_kernel<__nv_bfloat16, 0>),
                allow_big_cluster(quant_fused_kernel<float, 0>),
                allow_big_cluster(quant_fused_kernel<__nv_bfloat16, 1>),
                allow_big_cluster(rmsnorm_quant_kernel),
            };
            for (cudaError_t x : es)
                if (x != cudaSuccess) return cuda_fail(x, "cudaFuncSetAttribute");
            unsigned long long t = (unsigned long long)g_opt_timeout_ns;
            if ((e = cudaMemcpyToSymbol(g_timeout_ns, &t, sizeof t)) != cudaSuccess)
                return cuda_fail(e, "cudaMemcpyToSymbol(timeout)");
            d.ready.store(true, std::memory_order_release);
        }
    }
    *out = &d;
    return NVFP4SK_OK;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                   Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (g_opt_pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cluster > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = cluster;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

int launched(cudaError_t e, const char *what)
{
    if (e != cudaSuccess) return cuda_fail(e, what);
    return NVFP4SK_OK;
}

// ---- tensor maps (driver entry point fetched through the runtime) ---------
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

PFN_encodeTiled_t encode_fn()
{
    static PFN_encodeTiled_t fn = []() -> PFN_encodeTiled_t {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_encodeTiled_t>(p);
    }();
    return fn;
}

// 2-D byte tensor [rows][inner] with row stride `stride`, box [box_rows][box_inner]
int make_map_u8(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t stride, uint32_t box_inner,
                uint32_t box_rows, CUtensorMapSwizzle swz)
{
    PFN_encodeTiled_t fn = encode_fn();
    if (!fn) return fail(NVFP4SK_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {stride};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4SK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return NVFP4SK_OK;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- sizes shared by the workspace queries and the calls -------------------
int linear_grid(const DevInfo &d, int64_t U)
{
    int64_t G = g_opt_linear_ctas > 0 ? g_opt_linear_ctas : d.sms;
    return (int)std::min<int64_t>(G, U);
}
// Linear workspace: arrival counters int32 [NT][4] at offset 0 (fixed
// capacity, so that calls of any shape agree on where they live), then the
// split-K partial tiles fp32 [G][2][16][128].
constexpr int64_t LIN_MAX_NT = 4096;
constexpr size_t LIN_COUNTER_BYTES = LIN_MAX_NT * 4 * 4;
size_t linear_ws(int64_t G, int64_t NT) { (void)NT; return LIN_COUNTER_BYTES + up256((size_t)G * 2 * 16 * 128 * 4); }
// gate+up with SwiGLU: the same counters, partial tiles of gate and up, fp32 [G][2][128][32]
size_t linear_sw_ws(int64_t G) { return LIN_COUNTER_BYTES + up256((size_t)G * 2 * 32 * 128 * 4); }

int attn_splits(const DevInfo &d, int Hkv, int64_t n_log)
{
    int64_t S = g_opt_attn_splits > 0 ? g_opt_attn_splits : std::max<int64_t>(1, d.sms / std::max(1, Hkv));
    return (int)std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(S, ATT_MAX_SPLITS), n_log));
}
// Attention workspace: per-CTA-head arrival counters of the fused combine at
// offset 0 (ATT_CNT_BYTES), then the split results: o fp32
// [heads][S][rows_cta][128] and (m, l) fp32 [heads][S][rows_cta][2].  Tree
// mode: heads = Hkv, rows_cta = group*16; causal mode: heads = Hq, rows_cta = 128.
size_t attn_ws(int heads, int S, int rows_cta)
{
    const size_t rows = (size_t)heads * S * rows_cta;
    return ATT_CNT_BYTES + up256(rows * ATT_D * 4) + up256(rows * 2 * 4);
}

int argmax_chunks(int64_t n) { return (int)std::max<int64_t>(1, std::min<int64_t>(64, n / 4096)); }

// Shared launch of the attention kernel (tree or causal mode, see attn.cuh)
// after the entry points' argument checks.
int attn_launch(const void *q, int64_t ld_q, int T, int Hq, int Hkv, const uint8_t *k_pool, const uint8_t *v_pool,
                int64_t n_pool_pages, const int32_t *page_table, int64_t ctx_len, const int32_t *parent,
                const float *k_scale, const float *v_scale, float sm_scale, void *out, const float *g_act,
                uint8_t *act_prepared, void *ws, size_t ws_bytes, nvfp4sk_stream_t stream, int causal)
{
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int64_t n_log = cdiv(ctx_len + T, ATT_P);
    const int group = Hq / Hkv;
    const int heads = causal ? Hq : Hkv;                      // grid.y
    const int rows_w = causal ? ATT_ROWS : 16, nheads = causal ? 1 : group;
    const int S = attn_splits(*d, heads, n_log);
    const size_t need = attn_ws(heads, S, nheads * rows_w);
    if (!ws || ws_bytes < need || !al16(ws))
        return fail(NVFP4SK_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned)", need);
    CUtensorMap tk;
    if (int rc = make_map_u8(&tk, k_pool, ATT_D, (uint64_t)n_pool_pages * Hkv * ATT_P, ATT_D, ATT_D, ATT_P,
                             CU_TENSOR_MAP_SWIZZLE_128B))
        return rc;
    AttnParams p;
    p.q = (const __nv_bfloat16 *)q;
    p.ld_q = ld_q;
    p.v_pool = v_pool;
    p.page_table = page_table;
    p.parent = parent;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.cnt = (int *)ws;
    p.part_o = (float *)((uint8_t *)ws + ATT_CNT_BYTES);
    p.part_ml = (float *)((uint8_t *)ws + ATT_CNT_BYTES + up256((size_t)heads * S * nheads * rows_w * ATT_D * 4));
    p.out = (__nv_bfloat16 *)out;
    p.g_act = g_act;
    p.act = act_prepared;
    p.ctx_len = ctx_len;
    p.n_pool_pages = n_pool_pages;
    p.sm_scale = sm_scale;
    p.T = T;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.group = group;
    p.S = S;
    p.n_log_pages = (int)n_log;
    p.causal = causal;
    p.rows_w = rows_w;
    p.nheads = nheads;
    // fused combine (on request) when every CTA of the grid can be resident at
    // once (one CTA per SM): the CTAs of a head wait for each other before
    // merging.  Measured on B200 at the verify step's shape: 27.2 us per call
    // fused against 24.6 us with the separate combine launch, so off by default.
    p.fuse = (g_opt_attn_fused && (int64_t)S * heads <= d->sms) ? 1 : 0;
    cudaStream_t st = (cudaStream_t)stream;
    // split results: fp32 rows of 512 bytes, one TMA box = 128 bytes (32 dims) x the CTA's rows
    CUtensorMap to;
    if (int rc = make_map_u8(&to, p.part_o, ATT_D * 4, (uint64_t)heads * S * nheads * rows_w, ATT_D * 4, 128,
                             (uint32_t)(nheads * rows_w), CU_TENSOR_MAP_SWIZZLE_128B))
        return rc;
    cudaError_t e = launch(tree_attn_split_kernel, dim3(S, heads), dim3(ATT_THREADS), ATT_SMEM_BYTES, st, 1, tk, to, p);
    if (e != cudaSuccess) return cuda_fail(e, "tree_attn_split_kernel");
    if (p.fuse) return NVFP4SK_OK;
    return launched(launch(tree_attn_combine_kernel, dim3(T, Hq), dim3(ATT_D), 0, st, 1, p),
                    "tree_attn_combine_kernel");
}


}  // namespace

// ============================================================================
extern "C" {

int nvfp4sk_version(void) { return 100; }
const char *nvfp4sk_last_error(void) { return t_last_error.c_str(); }

nvfp4sk_status nvfp4sk_set_option(int option, int64_t value)
{
    switch (option) {
    case NVFP4SK_OPT_PDL: g_opt_pdl = value ? 1 : 0; return NVFP4SK_OK;
    case NVFP4SK_OPT_TIMEOUT_NS: {
        if (value <= 0) return fail(NVFP4SK_ERR_INVALID_ARG, "timeout must be positive");
        g_opt_timeout_ns = value;
        unsigned long long t = (unsigned long long)value;
        cudaError_t e = cudaMemcpyToSymbol(g_timeout_ns, &t, sizeof t);
        return e == cudaSuccess ? NVFP4SK_OK : cuda_fail(e, "cudaMemcpyToSymbol(timeout)");
    }
    case NVFP4SK_OPT_ATTN_SPLITS: g_opt_attn_splits = (int)std::max<int64_t>(0, value); return NVFP4SK_OK;
    case NVFP4SK_OPT_LINEAR_CTAS: g_opt_linear_ctas = (int)std::max<int64_t>(0, value); return NVFP4SK_OK;
    case NVFP4SK_OPT_ATTN_FUSED_COMBINE: g_opt_attn_fused = value ? 1 : 0; return NVFP4SK_OK;
    default: return fail(NVFP4SK_ERR_INVALID_ARG, "unknown option %d", option);
    }
}

int64_t nvfp4sk_get_option(int option)
{
    switch (option) {
    case NVFP4SK_OPT_PDL: return g_opt_pdl;
    case NVFP4SK_OPT_TIMEOUT_NS: return g_opt_timeout_ns;
    case NVFP4SK_OPT_ATTN_SPLITS: return g_opt_attn_splits;
    case NVFP4SK_OPT_LINEAR_CTAS: return g_opt_linear_ctas;
    case NVFP4SK_OPT_ATTN_FUSED_COMBINE: return g_opt_attn_fused;
    default: return -1;
    }
}

nvfp4sk_status nvfp4sk_get_device_status(nvfp4sk_stream_t stream, int *site)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int err = 0, where = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&err, g_err, sizeof err)) != cudaSuccess) return cuda_fail(e, "read status");
    cudaMemcpyFromSymbol(&where, g_err_site, sizeof where);
    cudaMemcpyToSymbol(g_err, &zero, sizeof zero);
    cudaMemcpyToSymbol(g_err_site, &zero, sizeof zero);
    if (site) *site = (int)where;
    if (err & ERRBIT_TIMEOUT) return fail(NVFP4SK_ERR_TIMEOUT, "device wait ran out (site %u)", where);
    if (err & ERRBIT_RANGE) return fail(NVFP4SK_ERR_OUT_OF_RANGE, "device bounds check failed (site %u)", where);
    return NVFP4SK_OK;
}

// ---------------------------------------------------------------- quantise
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K)
{
    (void)rows; (void)K;
    return QBIG_MAX_PARTIALS * sizeof(float);
}

size_t nvfp4_prepared_act_bytes(int64_t K) { return (size_t)cdiv(K, LIN_KC) * LIN_A_UNIT; }

nvfp4sk_status nvfp4_quantize_act(const void *x, int x_dtype, int64_t rows, int64_t K, int64_t ld_x,
                                  const float *g_in, uint8_t *codes, uint8_t *scales, float *g_out,
                                  uint8_t *act_prepared, void *ws, size_t ws_bytes, nvfp4sk_stream_t stream)
{
    if (!x || !g_out || (!act_prepared && (!codes || !scales)))
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer (need codes+scales and/or act_prepared)");
    if (x_dtype != NVFP4SK_BF16 && x_dtype != NVFP4SK_FP32) return fail(NVFP4SK_ERR_INVALID_ARG, "bad dtype");
    if (rows < 1 || K < 16 || K % 16 != 0 || ld_x < K)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need rows >= 1, K %% 16 == 0, ld_x >= K");
    if (act_prepared && (rows > 16 || K % 64 != 0))
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "the prepared activation needs rows <= 16 and K %% 64 == 0");
    const int64_t esz = x_dtype == NVFP4SK_BF16 ? 2 : 4;
    if (!al16(x) || (ld_x * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(codes) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(act_prepared) & 15u) != 0)
        return fail(NVFP4SK_ERR_MISALIGNED,
                    "x, its row stride and act_prepared must be 16-byte aligned, codes 8-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t nblk = rows * (K / 16);
    if (nblk <= QSMALL_MAX_BLOCKS && !g_in) {
        const int cs = nblk <= (int64_t)8 * QTHREADS * QNB ? 8 : 16;
        cudaError_t e = x_dtype == NVFP4SK_BF16
                            ? launch(quant_fused_kernel<__nv_bfloat16, 0>, dim3(cs), dim3(QTHREADS), 0, st, cs,
                                     (const __nv_bfloat16 *)x, rows, K, ld_x, g_in, codes, scales, g_out,
                                     act_prepared)
                            : launch(quant_fused_kernel<float, 0>, dim3(cs), dim3(QTHREADS), 0, st, cs,
                                     (const float *)x, rows, K, ld_x, g_in, codes, scales, g_out, act_prepared);
        return launched(e, "quant_fused_kernel");
    }
    if (!g_in && (!ws || ws_bytes < nvfp4_quantize_workspace_bytes(rows, K)))
        return fail(NVFP4SK_ERR_WORKSPACE, "workspace too small");
    // one thread per 16-block with a static scale; with a dynamic one the grid
    // is capped by the amax partials it leaves
    const int grid = g_in ? (int)std::min<int64_t>(INT32_MAX, cdiv(nblk, QBIG_THREADS))
                          : (int)std::min<int64_t>(std::min<int64_t>(QBIG_MAX_PARTIALS, 4 * d->sms),
                                                   cdiv(nblk, QBIG_THREADS));
    float *partial = (float *)ws;
    cudaError_t e = cudaSuccess;
    if (!g_in) {
        e = x_dtype == NVFP4SK_BF16
                ? launch(amax_partial_kernel<__nv_bfloat16>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1,
                         (const __nv_bfloat16 *)x, rows, K, ld_x, partial)
                : launch(amax_partial_kernel<float>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1, (const float *)x,
                         rows, K, ld_x, partial);
        if (e != cudaSuccess) return cuda_fail(e, "amax_partial_kernel");
    }
    e = x_dtype == NVFP4SK_BF16
            ? launch(quant_blocks_kernel<__nv_bfloat16>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1,
                     (const __nv_bfloat16 *)x, rows, K, ld_x, g_in, (const float *)partial, grid, codes, scales,
                     g_out, act_prepared, (uint8_t *)nullptr)
            : launch(quant_blocks_kernel<float>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1, (const float *)x, rows,
                     K, ld_x, g_in, (const float *)partial, grid, codes, scales, g_out, act_prepared,
                     (uint8_t *)nullptr);
    return launched(e, "quant_blocks_kernel");
}

// ---- quantisers writing the wide linear's tile image (static scale) --------
static nvfp4sk_status tiles_check(const float *g_in, const float *g_out, const uint8_t *tiles, int64_t rows,
                                  int64_t K)
{
    if (!g_in || !g_out || !tiles) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer (the tile image needs g_in)");
    if (rows < 1 || rows > INT32_MAX || K < LIN_KC || K % LIN_KC != 0)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need rows >= 1, K %% 512 == 0");
    if (!al16(tiles)) return fail(NVFP4SK_ERR_MISALIGNED, "tiles must be 16-byte aligned");
    return NVFP4SK_OK;
}

nvfp4sk_status nvfp4_quantize_act_tiles(const void *x, int x_dtype, int64_t rows, int64_t K, int64_t ld_x,
                                        const float *g_in, float *g_out, uint8_t *tiles, nvfp4sk_stream_t stream)
{
    if (!x) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (x_dtype != NVFP4SK_BF16 && x_dtype != NVFP4SK_FP32) return fail(NVFP4SK_ERR_INVALID_ARG, "bad dtype");
    if (int rc = tiles_check(g_in, g_out, tiles, rows, K)) return rc;
    if (ld_x < K) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need ld_x >= K");
    const int64_t esz = x_dtype == NVFP4SK_BF16 ? 2 : 4;
    if (!al16(x) || (ld_x * esz) % 16 != 0) return fail(NVFP4SK_ERR_MISALIGNED, "x and its row stride must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    const int grid = (int)std::min<int64_t>(INT32_MAX, cdiv(rows * (K / 16), QBIG_THREADS));
    uint8_t *none = nullptr;
    cudaError_t e = x_dtype == NVFP4SK_BF16
                        ? launch(quant_blocks_kernel<__nv_bfloat16>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1,
                                 (const __nv_bfloat16 *)x, rows, K, ld_x, g_in, (const float *)nullptr, 0, none, none,
                                 g_out, none, tiles)
                        : launch(quant_blocks_kernel<float>, dim3(grid), dim3(QBIG_THREADS), 0, st, 1, (const float *)x,
                                 rows, K, ld_x, g_in, (const float *)nullptr, 0, none, none, g_out, none, tiles);
    return launched(e, "quant_blocks_kernel (tile image)");
}

nvfp4sk_status nvfp4_rmsnorm_quantize_tiles(const void *x, const void *w, float eps, int64_t rows, int64_t n,
                                            const float *g_in, float *g_out, uint8_t *tiles, nvfp4sk_stream_t stream)
{
    if (!x || !w) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (int rc = tiles_check(g_in, g_out, tiles, rows, n)) return rc;
    if (n > (int64_t)RTHREADS * RNB * 16) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need n <= 8192");
    if (!al16(x) || !al16(w)) return fail(NVFP4SK_ERR_MISALIGNED, "x and w must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    uint8_t *none = nullptr;
    return launched(launch(rmsnorm_quant_static_kernel, dim3((unsigned)rows, rows >= d->sms ? 1 : RS_SPLIT),
                           dim3(RS_THREADS), 0, (cudaStream_t)stream, 1, (const __nv_bfloat16 *)x,
                           (const __nv_bfloat16 *)w, eps, n, g_in, none, none, g_out, none, tiles),
                    "rmsnorm_quant_static_kernel (tile image)");
}

nvfp4sk_status nvfp4_swiglu_quantize_tiles(const void *gu, int64_t rows, int64_t F, const float *g_in, float *g_out,
                                           uint8_t *tiles, nvfp4sk_stream_t stream)
{
    if (!gu) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (int rc = tiles_check(g_in, g_out, tiles, rows, F)) return rc;
    if (!al16(gu)) return fail(NVFP4SK_ERR_MISALIGNED, "gu must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    uint8_t *none = nullptr;
    return launched(launch(swiglu_quant_static_kernel,
                           dim3((unsigned)std::min<int64_t>(INT32_MAX, cdiv(rows * (F / 16), QBIG_THREADS_STATIC))),
                           dim3(QBIG_THREADS_STATIC), 0, (cudaStream_t)stream, 1, (const __nv_bfloat16 *)gu, rows, F,
                           g_in, none, none, g_out, none, tiles),
                    "swiglu_quant_static_kernel (tile image)");
}

nvfp4sk_status nvfp4_prepare_act(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                                 uint8_t *act_prepared, nvfp4sk_stream_t stream)
{
    if (!codes || !scales || !act_prepared) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (rows < 1 || rows > 16 || K < 64 || K % 64 != 0)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= rows <= 16, K %% 64 == 0");
    if ((reinterpret_cast<uintptr_t>(codes) & 7u) || (reinterpret_cast<uintptr_t>(act_prepared) & 15u))
        return fail(NVFP4SK_ERR_MISALIGNED, "codes 8-byte aligned, act_prepared 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int64_t nblk = rows * (K / 16);
    const int grid = (int)std::min<int64_t>(cdiv(nblk, 256), 4 * d->sms);
    return launched(launch(prepare_act_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, 1, codes, scales, rows,
                           K, act_prepared),
                    "prepare_act_kernel");
}

size_t nvfp4_prepared_weight_bytes(int64_t N, int64_t K) { return (size_t)cdiv(N, 128) * cdiv(K, LIN_KC) * LIN_W_UNIT; }

nvfp4sk_status nvfp4_prepare_weight(const uint8_t *codes, const uint8_t *scales, int64_t N, int64_t K,
                                    uint8_t *prepared, nvfp4sk_stream_t stream)
{
    if (!codes || !scales || !prepared) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (N < 1 || K < 64 || K % 64 != 0) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need N >= 1, K %% 64 == 0");
    if (!al16(prepared) || !al16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return fail(NVFP4SK_ERR_MISALIGNED, "prepared and codes must be 16-byte aligned, scales 4-byte aligned");
    const int64_t units = cdiv(N, 128) * cdiv(K, LIN_KC);
    if (units > INT32_MAX) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "matrix too large");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(prepare_weight_kernel, dim3((unsigned)units), dim3(256), 0, (cudaStream_t)stream, 1, codes,
                           scales, N, K, cdiv(K, LIN_KC), prepared),
                    "prepare_weight_kernel");
}

// ---------------------------------------------------------------- linear
size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    (void)M;
    DevInfo *d;
    if (device_info(&d)) return 0;
    const int64_t NT = cdiv(N, 128), KC = cdiv(K, LIN_KC);
    const int64_t G = std::max<int64_t>(d->sms, g_opt_linear_ctas);
    return linear_ws(std::min<int64_t>(G, NT * KC), NT);
}

nvfp4sk_status nvfp4_linear(const uint8_t *a_prepared, const float *g_a, int64_t M, const uint8_t *w_prepared,
                            const float *g_w, int64_t N, int64_t K, const void *residual, void *y, int64_t ldy,
                            void *ws, size_t ws_bytes, nvfp4sk_stream_t stream)
{
    if (!a_prepared || !g_a || !w_prepared || !g_w || !y) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (M < 1 || M > 16 || N < 1 || N > LIN_MAX_NT * 128 || K < 64 || K % 64 != 0 || ldy < N)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= M <= 16, 1 <= N <= 524288, K %% 64 == 0, ldy >= N");
    if (!al16(a_prepared) || !al16(w_prepared))
        return fail(NVFP4SK_ERR_MISALIGNED, "prepared operands must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int64_t NT = cdiv(N, 128), KC = cdiv(K, LIN_KC), U = NT * KC;
    const int G = linear_grid(*d, U);
    const size_t need = linear_ws(G, NT);
    if (!ws || ws_bytes < need || !al16(ws))
        return fail(NVFP4SK_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned)", need);
    LinearParams p;
    p.w = w_prepared;
    p.a = a_prepared;
    p.g_a = g_a;
    p.g_w = g_w;
    p.residual = (const __nv_bfloat16 *)residual;
    p.y = (__nv_bfloat16 *)y;
    p.counters = (int *)ws;
    p.partial = (float *)((uint8_t *)ws + LIN_COUNTER_BYTES);
    p.ldy = ldy;
    p.U = U;
    p.M = (int)M;
    p.N = (int)N;
    p.NT = (int)NT;
    p.KC = (int)KC;
    p.sw_act = nullptr;
    p.sw_g = nullptr;
    return launched(launch(nvfp4_linear_kernel<false>, dim3(G), dim3(LIN_THREADS), LIN_SMEM_BYTES, (cudaStream_t)stream, 1,
                           p),
                    "nvfp4_linear_kernel");
}

size_t nvfp4_linear_swiglu_workspace_bytes(int64_t M, int64_t F, int64_t K)
{
    (void)M;
    DevInfo *d;
    if (device_info(&d)) return 0;
    const int64_t NT = cdiv(F, 128), KC = cdiv(K, LIN_KC);
    const int64_t G = std::max<int64_t>(d->sms, g_opt_linear_ctas);
    return linear_sw_ws(std::max<int64_t>(1, std::min<int64_t>(G, NT * KC)));
}

nvfp4sk_status nvfp4_linear_swiglu(const uint8_t *a_prepared, const float *g_a, int64_t M, const uint8_t *w_prepared,
                                   const float *g_w, int64_t F, int64_t K, const float *g_out, uint8_t *act_out,
                                   void *ws, size_t ws_bytes, nvfp4sk_stream_t stream)
{
    if (!a_prepared || !g_a || !w_prepared || !g_w || !g_out || !act_out)
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (M < 1 || M > 16 || F < 128 || F % 128 != 0 || F > LIN_MAX_NT * 128 || K < 64 || K % 64 != 0)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= M <= 16, F %% 128 == 0 (128 <= F <= 524288), K %% 64 == 0");
    if (!al16(a_prepared) || !al16(w_prepared) || !al16(act_out))
        return fail(NVFP4SK_ERR_MISALIGNED, "prepared operands and act_out must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int64_t NT = F / 128, KC = cdiv(K, LIN_KC), U = NT * KC;
    const int G = linear_grid(*d, U);
    const size_t need = linear_sw_ws(G);
    if (!ws || ws_bytes < need || !al16(ws))
        return fail(NVFP4SK_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned)", need);
    LinearParams p;
    p.w = w_prepared;
    p.a = a_prepared;
    p.g_a = g_a;
    p.g_w = g_w;
    p.residual = nullptr;
    p.y = nullptr;
    p.counters = (int *)ws;
    p.partial = (float *)((uint8_t *)ws + LIN_COUNTER_BYTES);
    p.ldy = 0;
    p.U = U;
    p.M = (int)M;
    p.N = (int)F;
    p.NT = (int)NT;
    p.KC = (int)KC;
    p.sw_act = act_out;
    p.sw_g = g_out;
    return launched(launch(nvfp4_linear_kernel<true>, dim3(G), dim3(LIN_THREADS), LIN_SMEM_BYTES_SW,
                           (cudaStream_t)stream, 1, p),
                    "nvfp4_linear_kernel (gate+up, SwiGLU)");
}

nvfp4sk_status nvfp4_linear_wide(const uint8_t *a_prepared, const float *g_a, int64_t S, const uint8_t *w_prepared,
                                 const float *g_w, int64_t N, int64_t K, const void *residual, void *y, int64_t ldy,
                                 nvfp4sk_stream_t stream)
{
    if (!a_prepared || !g_a || !w_prepared || !g_w || !y) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (S < 1 || S > INT32_MAX / 2 || N < 1 || N > INT32_MAX / 2 || K < 64 || K % 64 != 0 || ldy < N)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need S >= 1, N >= 1, K %% 64 == 0, ldy >= N");
    if (!al16(a_prepared) || !al16(w_prepared))
        return fail(NVFP4SK_ERR_MISALIGNED, "prepared operands must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    WideParams p;
    p.w = w_prepared;
    p.a = a_prepared;
    p.g_a = g_a;
    p.g_w = g_w;
    p.residual = (const __nv_bfloat16 *)residual;
    p.y = (__nv_bfloat16 *)y;
    p.ldy = ldy;
    p.S = S;
    p.N = N;
    p.NT = (int)cdiv(N, 128);
    p.ST = (int)cdiv(S, 128);
    p.KC = (int)cdiv(K, LIN_KC);
    const int64_t tiles = (int64_t)p.NT * ((p.ST + 1) / 2);
    if (tiles > INT32_MAX) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "too many output tiles");
    p.n_tiles = (int)tiles;
    const int G = (int)std::min<int64_t>(d->sms, tiles);
    return launched(launch(nvfp4_linear_wide_kernel, dim3(G), dim3(WD_THREADS), WD_SMEM_BYTES, (cudaStream_t)stream, 1, p),
                    "nvfp4_linear_wide_kernel");
}

// ---------------------------------------------------------------- attention
size_t tree_attn_workspace_bytes(int T, int Hq, int Hkv, int D, int page_size, int64_t ctx_len)
{
    (void)D;
    DevInfo *d;
    if (device_info(&d) || Hkv <= 0 || page_size <= 0 || Hq % Hkv) return 0;
    const int64_t n_log = cdiv(ctx_len + T, page_size);
    return attn_ws(Hkv, attn_splits(*d, Hkv, n_log), Hq / Hkv * 16);
}

size_t causal_attn_workspace_bytes(int T, int Hq, int Hkv, int D, int page_size, int64_t ctx_len)
{
    (void)D; (void)Hkv;
    DevInfo *d;
    if (device_info(&d) || Hq <= 0 || page_size <= 0) return 0;
    const int64_t n_log = cdiv(ctx_len + T, page_size);
    return attn_ws(Hq, attn_splits(*d, Hq, n_log), ATT_ROWS);
}

nvfp4sk_status tree_attn_fp8kv(const void *q, int64_t ld_q, int T, int Hq, int Hkv, int D, const uint8_t *k_pool,
                               const uint8_t *v_pool, int64_t n_pool_pages, int page_size,
                               const int32_t *page_table, int64_t ctx_len, const int32_t *parent,
                               const float *k_scale, const float *v_scale, float sm_scale, void *out,
                               const float *g_act, uint8_t *act_prepared, void *ws, size_t ws_bytes,
                               nvfp4sk_stream_t stream)
{
    if (!q || !k_pool || !v_pool || !page_table || !parent || !k_scale || !v_scale || !out)
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (D != ATT_D || page_size != ATT_P || T < 1 || T > ATT_T || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > 8 ||
        ctx_len < 0 || n_pool_pages < 1 || ld_q < (int64_t)Hq * D || n_pool_pages * Hkv * ATT_P > INT32_MAX)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "need D == 128, page_size == 64, 1 <= T <= 16, Hq %% Hkv == 0, Hq/Hkv <= 8, ld_q >= Hq*D");
    if (!al16(q) || ld_q % 8 != 0 || !al16(k_pool) || !al16(v_pool) || !al16(act_prepared))
        return fail(NVFP4SK_ERR_MISALIGNED, "q (and ld_q*2 bytes), the pools and act_prepared must be 16-byte aligned");
    if (act_prepared && !g_act) return fail(NVFP4SK_ERR_INVALID_ARG, "act_prepared needs the static scale g_act");
    return attn_launch(q, ld_q, T, Hq, Hkv, k_pool, v_pool, n_pool_pages, page_table, ctx_len, parent, k_scale,
                       v_scale, sm_scale, out, g_act, act_prepared, ws, ws_bytes, stream, 0);
}

nvfp4sk_status causal_attn_fp8kv(const void *q, int64_t ld_q, int T, int Hq, int Hkv, int D, const uint8_t *k_pool,
                                 const uint8_t *v_pool, int64_t n_pool_pages, int page_size,
                                 const int32_t *page_table, int64_t ctx_len, const float *k_scale,
                                 const float *v_scale, float sm_scale, void *out, void *ws, size_t ws_bytes,
                                 nvfp4sk_stream_t stream)
{
    if (!q || !k_pool || !v_pool || !page_table || !k_scale || !v_scale || !out)
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (D != ATT_D || page_size != ATT_P || T < 1 || T > ATT_ROWS || Hkv < 1 || Hq % Hkv != 0 ||
        Hq * 4 > (int)ATT_CNT_BYTES || ctx_len < 0 || n_pool_pages < 1 || ld_q < (int64_t)Hq * D ||
        n_pool_pages * Hkv * ATT_P > INT32_MAX)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "need D == 128, page_size == 64, 1 <= T <= 128, Hq %% Hkv == 0, Hq <= 64, ld_q >= Hq*D");
    if (!al16(q) || ld_q % 8 != 0 || !al16(k_pool) || !al16(v_pool))
        return fail(NVFP4SK_ERR_MISALIGNED, "q (and ld_q*2 bytes) and the pools must be 16-byte aligned");
    return attn_launch(q, ld_q, T, Hq, Hkv, k_pool, v_pool, n_pool_pages, page_table, ctx_len, nullptr, k_scale,
                       v_scale, sm_scale, out, nullptr, nullptr, ws, ws_bytes, stream, 1);
}

// ---------------------------------------------------------------- restore
nvfp4sk_status kv_page_restore(const uint8_t *src_pool, const int32_t *src_ids, uint8_t *dst_pool,
                               const int32_t *dst_ids, int64_t n, int64_t page_bytes, int64_t n_src_pages,
                               int64_t n_dst_pages, nvfp4sk_stream_t stream)
{
    if (n == 0) return NVFP4SK_OK;
    if (!src_pool || !src_ids || !dst_pool || !dst_ids) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (n < 0 || page_bytes < 16 || page_bytes % 16 != 0 || n_src_pages < 1 || n_dst_pages < 1)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need n >= 0, page_bytes %% 16 == 0");
    if (!al16(src_pool) || !al16(dst_pool)) return fail(NVFP4SK_ERR_MISALIGNED, "pools must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    RestoreParams p;
    p.src = src_pool;
    p.src_ids = src_ids;
    p.dst = dst_pool;
    p.dst_ids = dst_ids;
    p.page_bytes = page_bytes;
    p.n_src_pages = n_src_pages;
    p.n_dst_pages = n_dst_pages;
    p.chunk = (uint32_t)std::min<int64_t>(page_bytes, 32768);
    p.chunks_per_page = (int)cdiv(page_bytes, p.chunk);
    p.n_items = n * p.chunks_per_page;
    p.stages = (int)std::max<uint32_t>(2, std::min<uint32_t>(RST_MAX_STAGES, RST_SMEM_BUDGET / p.chunk));
    const size_t smem = (size_t)p.stages * p.chunk + 128 + 8 * RST_MAX_STAGES + 64;
    const int grid = (int)std::min<int64_t>(p.n_items, d->sms);
    return launched(launch(kv_page_restore_kernel, dim3(grid), dim3(RST_THREADS), smem, (cudaStream_t)stream, 1, p),
                    "kv_page_restore_kernel");
}

// ---------------------------------------------------------------- glue
nvfp4sk_status nvfp4_rmsnorm_quantize(const void *x, const void *w, float eps, int64_t rows, int64_t n,
                                      const float *g_in, uint8_t *codes, uint8_t *scales, float *g_out,
                                      uint8_t *act_prepared, void *ws, size_t ws_bytes, nvfp4sk_stream_t stream)
{
    (void)ws; (void)ws_bytes;
    if (!x || !w || !g_out || (!act_prepared && (!codes || !scales)))
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    // the static-scale path with canonical outputs takes any row count (the
    // suffix prefill); the dynamic path and the 16-row prepared image do not
    const int64_t max_rows = (g_in && !act_prepared) ? (int64_t)INT32_MAX : 16;
    if (rows < 1 || rows > max_rows || n < 64 || n % 64 != 0 || n > (int64_t)RTHREADS * RNB * 16)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "need 1 <= rows <= 16 (any with g_in and no act_prepared), n %% 64 == 0, n <= 8192");
    if (!al16(x) || !al16(w) || (reinterpret_cast<uintptr_t>(codes) & 7u) ||
        (reinterpret_cast<uintptr_t>(act_prepared) & 15u))
        return fail(NVFP4SK_ERR_MISALIGNED, "x, w, act_prepared must be 16-byte aligned, codes 8-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    if (g_in)
        // RS_SPLIT CTAs per row while there are few rows; one per row once they fill the GPU
        return launched(launch(rmsnorm_quant_static_kernel, dim3((unsigned)rows, rows >= d->sms ? 1 : RS_SPLIT),
                               dim3(RS_THREADS), 0,
                               (cudaStream_t)stream, 1, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w, eps, n,
                               g_in, codes, scales, g_out, act_prepared, (uint8_t *)nullptr),
                        "rmsnorm_quant_static_kernel");
    const int cs = rows <= 8 ? 8 : 16;
    return launched(launch(rmsnorm_quant_kernel, dim3(cs), dim3(RTHREADS), 0, (cudaStream_t)stream, cs,
                           (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w, eps, rows, n, codes, scales, g_out,
                           act_prepared),
                    "rmsnorm_quant_kernel");
}

nvfp4sk_status nvfp4_swiglu_quantize(const void *gu, int64_t rows, int64_t F, const float *g_in, uint8_t *codes,
                                     uint8_t *scales, float *g_out, uint8_t *act_prepared, void *ws, size_t ws_bytes,
                                     nvfp4sk_stream_t stream)
{
    (void)ws; (void)ws_bytes;
    if (!gu || !g_out || (!act_prepared && (!codes || !scales)))
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    const bool any_rows = g_in && !act_prepared;        // static scale, canonical outputs: any row count
    if (rows < 1 || (!any_rows && (rows > 16 || rows * (F / 16) > QSMALL_MAX_BLOCKS)) || rows > INT32_MAX || F < 64 ||
        F % 64 != 0)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "need 1 <= rows <= 16 (any with g_in and no act_prepared), F %% 64 == 0, rows*F <= 524288");
    if (!al16(gu) || (reinterpret_cast<uintptr_t>(codes) & 7u) || (reinterpret_cast<uintptr_t>(act_prepared) & 15u))
        return fail(NVFP4SK_ERR_MISALIGNED, "gu, act_prepared must be 16-byte aligned, codes 8-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int64_t nblk = rows * (F / 16);
    if (g_in)
        return launched(launch(swiglu_quant_static_kernel,
                               dim3((unsigned)std::min<int64_t>(INT32_MAX, cdiv(nblk, QBIG_THREADS_STATIC))),
                               dim3(QBIG_THREADS_STATIC), 0, (cudaStream_t)stream, 1, (const __nv_bfloat16 *)gu, rows,
                               F, g_in, codes, scales, g_out, act_prepared, (uint8_t *)nullptr),
                        "swiglu_quant_static_kernel");
    const int cs = nblk <= (int64_t)8 * QTHREADS * QNB ? 8 : 16;
    return launched(launch(quant_fused_kernel<__nv_bfloat16, 1>, dim3(cs), dim3(QTHREADS), 0, (cudaStream_t)stream,
                           cs, (const __nv_bfloat16 *)gu, rows, F, 2 * F, (const float *)nullptr, codes, scales,
                           g_out, act_prepared),
                    "swiglu_quant_kernel");
}

nvfp4sk_status kv_append_fp8(const void *k_new, const void *v_new, int64_t ld_new, int T, int Hkv, int D,
                             uint8_t *k_pool, uint8_t *v_pool, int64_t n_pool_pages, int page_size,
                             const int32_t *page_table, int64_t ctx_len, const float *k_scale, const float *v_scale,
                             nvfp4sk_stream_t stream)
{
    if (!k_new || !v_new || !k_pool || !v_pool || !page_table || !k_scale || !v_scale)
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (T < 1 || Hkv < 1 || D < 8 || D % 8 || page_size < 16 || page_size % 16 || ctx_len < 0 ||
        ld_new < (int64_t)Hkv * D || n_pool_pages < 1)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need T, Hkv >= 1, D %% 8 == 0, page_size %% 16 == 0, ld_new >= Hkv*D");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(kv_append_kernel, dim3(T, Hkv), dim3(128), 0, (cudaStream_t)stream, 1,
                           (const __nv_bfloat16 *)k_new, (const __nv_bfloat16 *)v_new, ld_new, Hkv, D, k_pool,
                           v_pool, n_pool_pages, page_size, page_table, ctx_len, k_scale, v_scale),
                    "kv_append_kernel");
}

nvfp4sk_status kv_v_pages_to_tiled(const uint8_t *v_token_major, uint8_t *v_tiled, int64_t n_planes, int D,
                                   int page_size, nvfp4sk_stream_t stream)
{
    if (n_planes == 0) return NVFP4SK_OK;
    if (!v_token_major || !v_tiled) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (n_planes < 0 || n_planes > INT32_MAX || D < 8 || D % 8 || page_size < 16 || page_size % 16 ||
        (int64_t)D * page_size > KVT_MAX_PLANE)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need D %% 8 == 0, page_size %% 16 == 0, D*page_size <= %d",
                    KVT_MAX_PLANE);
    if (!al16(v_token_major) || !al16(v_tiled)) return fail(NVFP4SK_ERR_MISALIGNED, "planes must be 16-byte aligned");
    const uint8_t *a = v_token_major, *b = v_tiled;
    const int64_t total = n_planes * D * page_size;
    if (a < b + total && b < a + total) return fail(NVFP4SK_ERR_INVALID_ARG, "source and destination overlap");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(kv_v_to_tiled_kernel, dim3((unsigned)n_planes), dim3(256), 0, (cudaStream_t)stream, 1,
                           v_token_major, v_tiled, D, page_size),
                    "kv_v_to_tiled_kernel");
}

// Argmax workspace: arrival counters int32 [rows] at offset 0 (fixed
// capacity), then per-chunk values fp32 [rows][nch] and indices i32 [rows][nch].
constexpr int64_t AMX_MAX_ROWS = 4096;
constexpr size_t AMX_COUNTER_BYTES = AMX_MAX_ROWS * 4;
size_t argmax_workspace_bytes(int64_t rows, int64_t n)
{
    const int nch = argmax_chunks(n);
    return AMX_COUNTER_BYTES + up256((size_t)rows * nch * 4) * 2;
}

nvfp4sk_status argmax_rows_bf16(const void *x, int64_t rows, int64_t n, int64_t ld, int32_t *idx, void *ws,
                                size_t ws_bytes, nvfp4sk_stream_t stream)
{
    if (!x || !idx) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (rows < 1 || rows > AMX_MAX_ROWS || n < 1 || n > INT32_MAX || ld < n)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= rows <= 4096, ld >= n");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const size_t need = argmax_workspace_bytes(rows, n);
    if (!ws || ws_bytes < need) return fail(NVFP4SK_ERR_WORKSPACE, "workspace needs %zu bytes", need);
    const int nch = argmax_chunks(n);
    uint8_t *b = (uint8_t *)ws;
    int32_t *cnt = (int32_t *)b;
    float *pv = (float *)(b + AMX_COUNTER_BYTES);
    int32_t *pi = (int32_t *)(b + AMX_COUNTER_BYTES + up256((size_t)rows * nch * 4));
    return launched(launch(argmax_rows_kernel, dim3(nch, rows), dim3(AMX_THREADS), 0, (cudaStream_t)stream, 1,
                           (const __nv_bfloat16 *)x, n, ld, idx, pv, pi, cnt),
                    "argmax_rows_kernel");
}

nvfp4sk_status nvfp4sk_debug_encode(const float *x, int64_t n, uint8_t *e2m1, uint8_t *e4m3,
                                    nvfp4sk_stream_t stream)
{
    if (!x || n < 0) return fail(NVFP4SK_ERR_INVALID_ARG, "bad arguments");
    if (n == 0) return NVFP4SK_OK;
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    const int grid = (int)std::min<int64_t>(cdiv(n, 256), 16 * d->sms);
    return launched(launch(debug_encode_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, 1, x, n, e2m1, e4m3),
                    "debug_encode_kernel");
}

nvfp4sk_status tree_accept_greedy(const int32_t *draft_tokens, const int32_t *target_argmax, const int32_t *parent,
                                  int T, int32_t *path, int32_t *n_accepted, int32_t *next_token,
                                  nvfp4sk_stream_t stream)
{
    if (!draft_tokens || !target_argmax || !parent || !path || !n_accepted || !next_token)
        return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (T < 1 || T > ACC_MAX_T) return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= T <= 32");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(tree_accept_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream, 1, draft_tokens,
                           target_argmax, parent, T, path, n_accepted, next_token),
                    "tree_accept_kernel");
}

nvfp4sk_status kv_compact_accepted(uint8_t *k_pool, uint8_t *v_pool, int64_t layer_stride, int n_layers, int Hkv,
                                   int D, int64_t n_pool_pages, int page_size, const int32_t *page_table,
                                   int64_t ctx_len, const int32_t *path, const int32_t *n_accepted, int T,
                                   nvfp4sk_stream_t stream)
{
    if (!k_pool || !v_pool || !page_table || !path || !n_accepted) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (n_layers < 1 || Hkv < 1 || D < 8 || D > 128 || D % 8 || page_size < 16 || page_size % 16 || T < 1 ||
        T > ACC_MAX_T || ctx_len < 0 || n_pool_pages < 1 || layer_stride < 0)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "need n_layers, Hkv >= 1, 8 <= D <= 128, D %% 8 == 0, page_size %% 16 == 0, 1 <= T <= 32");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(kv_compact_kernel, dim3(n_layers, Hkv), dim3(128), 0, (cudaStream_t)stream, 1, k_pool,
                           v_pool, layer_stride, Hkv, D, n_pool_pages, page_size, page_table, ctx_len, path,
                           n_accepted, T),
                    "kv_compact_kernel");
}

nvfp4sk_status nvfp4sk_debug_wait_timeout(nvfp4sk_stream_t stream)
{
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    return launched(launch(debug_wait_timeout_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream, 1),
                    "debug_wait_timeout_kernel");
}

}  // extern "C"

// ============================================================================
// nvfp4_linear_noalloc: the NVFP4 linear for callers that cannot allocate.
//
// The scratch nvfp4_linear keeps in a caller-owned workspace (split-K arrival
// counters, partial tiles) lives here in one file-scope device array instead,
// sized for LIN_NOALLOC_MAX_CTAS CTAs and LIN_MAX_NT weight tiles.  The
// array's name is only a host-side stand-in: the device address is obtained
// with cudaGetSymbolAddress, once per device, on the first call made on that
// device.  Every call on a device shares the one array, so calls whose GPU
// work overlaps (different streams, no ordering) race on it.
// ============================================================================
namespace {
constexpr int LIN_NOALLOC_MAX_CTAS = 160;
constexpr size_t LIN_NOALLOC_SCRATCH_BYTES = LIN_COUNTER_BYTES + (size_t)LIN_NOALLOC_MAX_CTAS * 2 * 128 * 16 * 4;
}  // namespace

static __device__ __align__(256) uint8_t g_linear_noalloc_scratch[LIN_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array per device id; published with a release
// store once looked up, read with acquire loads (no lock on the fast path).
std::atomic<uint8_t *> g_noalloc_ptr[MAX_DEV];
std::mutex g_noalloc_mu;

int noalloc_scratch(uint8_t **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEV) return fail(NVFP4SK_ERR_DEVICE, "device id %d out of range", dev);
    uint8_t *p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            void *a = nullptr;
            e = cudaGetSymbolAddress(&a, g_linear_noalloc_scratch);
            if (e != cudaSuccess || !a) return cuda_fail(e, "cudaGetSymbolAddress(linear scratch)");
            p = (uint8_t *)a;
            g_noalloc_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return NVFP4SK_OK;
}
}  // namespace

extern "C" {

size_t nvfp4_linear_noalloc_scratch_bytes(void) { return LIN_NOALLOC_SCRATCH_BYTES; }

nvfp4sk_status nvfp4_linear_noalloc(const uint8_t *a_prepared, const float *g_a, int64_t M,
                                    const uint8_t *w_prepared, const float *g_w, int64_t N, int64_t K,
                                    const void *residual, void *y, int64_t ldy, nvfp4sk_stream_t stream)
{
    if (!a_prepared || !g_a || !w_prepared || !g_w || !y) return fail(NVFP4SK_ERR_INVALID_ARG, "null pointer");
    if (M < 1 || M > 16 || N < 1 || K < 64 || K % 64 != 0 || ldy < N)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE, "need 1 <= M <= 16, N >= 1, K %% 64 == 0, ldy >= N");
    if (N > LIN_MAX_NT * 128)
        return fail(NVFP4SK_ERR_UNSUPPORTED_SHAPE,
                    "N = %lld exceeds the built-in scratch of nvfp4_linear_noalloc (at most %lld output features)",
                    (long long)N, (long long)(LIN_MAX_NT * 128));
    if (!al16(a_prepared) || !al16(w_prepared))
        return fail(NVFP4SK_ERR_MISALIGNED, "prepared operands must be 16-byte aligned");
    DevInfo *d;
    if (int rc = device_info(&d)) return rc;
    uint8_t *scratch = nullptr;
    if (int rc = noalloc_scratch(&scratch)) return rc;
    const int64_t NT = cdiv(N, 128), KC = cdiv(K, LIN_KC), U = NT * KC;
    const int G = (int)std::min<int64_t>(std::min<int64_t>(linear_grid(*d, U), LIN_NOALLOC_MAX_CTAS), U);
    cudaStream_t st = (cudaStream_t)stream;
    // the arrival counters must read zero when the kernel starts
    cudaError_t e = cudaMemsetAsync(scratch, 0, (size_t)NT * 4 * sizeof(int), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(linear scratch counters)");
    LinearParams p;
    p.w = w_prepared;
    p.a = a_prepared;
    p.g_a = g_a;
    p.g_w = g_w;
    p.residual = (const __nv_bfloat16 *)residual;
    p.y = (__nv_bfloat16 *)y;
    p.counters = (int *)scratch;
    p.partial = (float *)(scratch + LIN_COUNTER_BYTES);
    p.ldy = ldy;
    p.U = U;
    p.M = (int)M;
    p.N = (int)N;
    p.NT = (int)NT;
    p.KC = (int)KC;
    p.sw_act = nullptr;
    p.sw_g = nullptr;
    return launched(launch(nvfp4_linear_kernel<false>, dim3(G), dim3(LIN_THREADS), LIN_SMEM_BYTES, st, 1, p),
                    "nvfp4_linear_kernel (no-alloc)");
}

}  // extern "C"
