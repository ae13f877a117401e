// wide.cuh -- NVFP4 (W4A4) linear layer for many tokens (the suffix prefill):
// Y[s][n] = g_a g_w sum_b s_a[s,b] s_w[n,b] sum_{k in b} a[s,k] w[n,k]
// (+ residual), fp32 accumulation, bf16 output, for S tokens at once.
//
// Same operand images as the skinny linear: the weight in 36 KB units (128
// rows x 512 K: two 16 KB 128-byte-swizzled code atoms, eight 512-byte scale
// images), and the activation in the same tile image with tokens as rows
// (nvfp4_prepare_weight applied to the S x K activation).
//
// Tile = 128 weight rows x 256 tokens, the whole K range in one CTA (no
// split-K: a prefill has hundreds of such tiles).  Per 512-K stage: one
// weight unit and the units of the two 128-token activation tiles, three
// 36 KB bulk copies (108 KB), two stages.  (Measured: shared memory fills
// from L2 at ~150 GB/s per SM with few large copies and ~85 GB/s with six
// copies of 16 KB and 2 KB per stage; the products of a stage need ~0.5 us.)
// Per 64-K step two tcgen05.mma.kind::mxf4nvf4.block_scale.block16 with
// M = 128 weight rows, N = 128 tokens each, into two fp32 accumulators of
// 128 columns in tensor memory.  The scale factors go to tensor memory with
// tcgen05.st from the epilogue warps (one warp per TMEM sub-partition), which
// keeps the tensor pipe free for the products.
// Tiles are numbered weight-tile-major (all token tiles of weight tile t,
// then t+1, ...) and dealt round-robin to a persistent grid, so the CTAs
// working at the same time share weight tiles through L2.
//
// Warp roles (192 threads, one CTA per SM): warp 0 producer (bulk copies),
// warp 1 TMEM allocation + MMA issue (one thread), warps 2-5 scale staging and
// the epilogue (tcgen05.ld, scale by g_a g_w, optional residual, bf16 store).
#pragma once
#include "common.cuh"
#include "linear.cuh"

namespace nvfp4sk {

constexpr int WD_STAGES = 2;
constexpr int WD_THREADS = 192;
constexpr uint32_t WD_STAGE_BYTES = 3 * LIN_W_UNIT;                // weights + two token tiles: 108 KB
constexpr uint32_t WD_OFF_BAR = WD_STAGES * WD_STAGE_BYTES;
constexpr uint32_t WD_SMEM_BYTES = WD_OFF_BAR + 256 + 1024;
constexpr uint32_t WD_TMEM_COLS = 512;
// TMEM columns: accumulators of token tiles 0 and 1 at 0 and 128; per stage s
// the weight scales (8 steps x 4 columns) at 256 + 32 s and the two token
// tiles' scales at 320 + 64 s (+32 for the second).
constexpr uint32_t WD_TM_ACC = 0, WD_TM_SFA = 256, WD_TM_SFB = 320;
static_assert(WD_TM_SFA + 32 * WD_STAGES <= WD_TM_SFB && WD_TM_SFB + 64 * WD_STAGES <= WD_TMEM_COLS,
              "tensor memory budget");
static_assert(WD_STAGE_BYTES % 1024 == 0, "swizzled code atoms need 1024-byte alignment");
static_assert(WD_SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct WideParams {
    const uint8_t *w;              // prepared weight units [NT][KC][36864]
    const uint8_t *a;              // prepared activation units [ST][KC][36864] (tokens as rows)
    const float *g_a;
    const float *g_w;
    const __nv_bfloat16 *residual; // nullable, [S][ldy]
    __nv_bfloat16 *y;              // [S][ldy]
    int64_t ldy;
    int64_t S, N;
    int NT, ST, KC;                // weight tiles, 128-token tiles, 512-K chunks
    int n_tiles;                   // NT * ceil(ST / 2)
};

__global__ void __launch_bounds__(WD_THREADS, 1) nvfp4_linear_wide_kernel(const WideParams p)
{
    extern __shared__ uint8_t wd_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(wd_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + WD_OFF_BAR);
    uint64_t *empty = full + WD_STAGES;
    uint64_t *sf_ready = empty + WD_STAGES;
    uint64_t *accf = sf_ready + WD_STAGES;
    uint64_t *acce = accf + 1;
    uint64_t *drain = acce + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int KH = p.KC;                           // 512-K steps per tile
    const int n_st2 = (p.ST + 1) / 2;              // 256-token tiles
    // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int my_tiles = p.n_tiles > (int)blockIdx.x ? (p.n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int64_t n_steps = (int64_t)my_tiles * KH;

    if (threadIdx.x == 0) {
        for (int s = 0; s < WD_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 4);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 4);
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, WD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();

    // tile k of this CTA -> (weight tile, first 128-token tile, has second token tile)
    auto tile_of = [&](int64_t k, int &tw, int &ts0, bool &two) {
        const int id = (int)blockIdx.x + (int)k * (int)gridDim.x;
        tw = id / n_st2;
        ts0 = 2 * (id % n_st2);
        two = ts0 + 1 < p.ST;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_last();    // a weight tile is read by every token tile
            const uint64_t pol_a = policy_evict_last();
            auto issue = [&](int64_t i) {
                const int s = (int)(i % WD_STAGES);
                int tw, ts0;
                bool two;
                tile_of(i / KH, tw, ts0, two);
                const int c = (int)(i % KH);
                uint8_t *dst = smem + s * WD_STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], (two ? 3u : 2u) * LIN_W_UNIT);
                bulk_load_hint(dst, p.w + ((int64_t)tw * p.KC + c) * LIN_W_UNIT, LIN_W_UNIT, &full[s], pol_w);
                for (int tt = 0; tt < (two ? 2 : 1); ++tt)
                    bulk_load_hint(dst + (1 + tt) * LIN_W_UNIT, p.a + ((int64_t)(ts0 + tt) * p.KC + c) * LIN_W_UNIT,
                                   LIN_W_UNIT, &full[s], pol_a);
            };
            pdl_wait();
            int64_t issued = 0;
            for (int64_t i = 0; i < n_steps; ++i) {
                if (i >= WD_STAGES &&
                    !mbar_wait(&empty[i % WD_STAGES], (uint32_t)(((i / WD_STAGES) - 1) & 1), 601, s_abort))
                    break;
                issue(i);
                issued = i + 1;
            }
            if (*s_abort) {
                for (int64_t i = issued > WD_STAGES ? issued - WD_STAGES : 0; i < issued; ++i)
                    mbar_wait_drain(&full[i % WD_STAGES], (uint32_t)((i / WD_STAGES) & 1), 602);
            }
        } else {
            pdl_wait();
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = lin_idesc(128, 128);
            bool ok = true;
            for (int64_t k = 0; k < my_tiles && ok; ++k) {
                int tw, ts0;
                bool two;
                tile_of(k, tw, ts0, two);
                if (!mbar_wait(acce, (uint32_t)((k & 1) ^ 1), 603, s_abort)) { ok = false; break; }
                tc_fence_after();
                for (int kh = 0; kh < KH; ++kh) {
                    const int64_t i = k * KH + kh;
                    const int s = (int)(i % WD_STAGES);
                    const uint32_t par = (uint32_t)((i / WD_STAGES) & 1);
                    if (!mbar_wait(&full[s], par, 604, s_abort) || !mbar_wait(&sf_ready[s], par, 605, s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * WD_STAGE_BYTES);
                    const uint32_t sfa_t = tmem_base + WD_TM_SFA + 32 * (uint32_t)s;
                    const uint32_t sfb_t = tmem_base + WD_TM_SFB + 64 * (uint32_t)s;
#pragma unroll
                    for (int j = 0; j < LIN_KSTEPS; ++j) {
                        const uint32_t ko = (uint32_t)(j >> 2) * LIN_W_ATOM + 32u * (uint32_t)(j & 3);
                        const uint64_t adesc = smem_desc(st + ko, 16, 1024, SWZ_128B);
#pragma unroll
                        for (int tt = 0; tt < 2; ++tt) {
                            if (tt == 1 && !two) break;
                            const uint64_t bdesc = smem_desc(st + (1 + tt) * LIN_W_UNIT + ko, 16, 1024, SWZ_128B);
                            mma_mxf4nvf4(tmem_base + WD_TM_ACC + 128 * tt, adesc, bdesc, idesc, sfa_t + 4 * j,
                                         sfb_t + 32 * tt + 4 * j, (kh > 0 || j > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(accf);
            }
            if (!ok) {
                tc_commit(drain);
                mbar_wait_drain(drain, 0, 606);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ scale staging + epilogue
        pdl_wait();
        const uint32_t q = warp & 3;
        const uint32_t lane_base = tmem_base + ((32u * q) << 16);
        const float gs = __fmul_rn(*p.g_a, *p.g_w);
        int64_t next_sf = 0;
        bool sf_ok = true;
        // the scale images of step i (eight 64-K images per 128-row tile, line l
        // = rows l, l+32, l+64, l+96) to every TMEM sub-partition, then one arrive
        auto stage_scales = [&](int64_t i) -> bool {
            const int s = (int)(i % WD_STAGES);
            const bool landed = mbar_wait(&full[s], (uint32_t)((i / WD_STAGES) & 1), 607, s_abort);
            if (!__all_sync(0xFFFFFFFFu, landed)) return false;
            const uint8_t *st = smem + s * WD_STAGE_BYTES;
#pragma unroll
            for (int part = 0; part < 3; ++part) {
                const uint8_t *img = st + part * LIN_W_UNIT + 2 * LIN_W_ATOM;
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < LIN_KSTEPS; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(img + LIN_SF_IMG * j + 16 * lane);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                const uint32_t col = part == 0 ? WD_TM_SFA + 32 * (uint32_t)s : WD_TM_SFB + 64 * (uint32_t)s + 32 * (part - 1);
                tmem_st_x32(lane_base + col, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sf_ready[s]);
            return true;
        };
        for (int64_t k = 0; k < my_tiles; ++k) {
            int tw, ts0;
            bool two;
            tile_of(k, tw, ts0, two);
            // stage the scales of this tile and of the first steps of the next
            const int64_t lim = (k + 1) * KH - 1 + (WD_STAGES - 1);
            while (sf_ok && next_sf <= lim && next_sf < n_steps) sf_ok = stage_scales(next_sf++);
            if (!sf_ok) break;
            bool ok = true;
            if (lane == 0) ok = mbar_wait(accf, (uint32_t)(k & 1), 608, s_abort);
            if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
            tc_fence_after();
            const int64_t n = (int64_t)tw * 128 + 32 * q + lane;      // weight row of this thread
            for (int tt = 0; tt < (two ? 2 : 1); ++tt) {
#pragma unroll 1
                for (int cb = 0; cb < 128; cb += 32) {
                    uint32_t r[32];
                    tmem_ld_x32(lane_base + WD_TM_ACC + 128 * tt + cb, r);
                    tmem_wait_ld();
                    const int64_t s0 = (int64_t)(ts0 + tt) * 128 + cb;
                    if (n < p.N) {
                        // y may alias the residual (y = h + linear(h)): all 32
                        // residual loads go out before the first store
                        if (p.residual) {
                            __nv_bfloat16 res[32];
#pragma unroll
                            for (int m = 0; m < 32; ++m)
                                res[m] = s0 + m < p.S ? p.residual[(s0 + m) * p.ldy + n] : __float2bfloat16_rn(0.f);
#pragma unroll
                            for (int m = 0; m < 32; ++m)
                                r[m] = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(r[m]), gs),
                                                                 __bfloat162float(res[m])));
                        } else {
#pragma unroll
                            for (int m = 0; m < 32; ++m) r[m] = __float_as_uint(__fmul_rn(__uint_as_float(r[m]), gs));
                        }
#pragma unroll
                        for (int m = 0; m < 32; ++m)
                            if (s0 + m < p.S) p.y[(s0 + m) * p.ldy + n] = __float2bfloat16_rn(__uint_as_float(r[m]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, WD_TMEM_COLS);
    }
}

}  // namespace nvfp4sk
