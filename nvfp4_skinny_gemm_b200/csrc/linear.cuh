// linear.cuh -- NVFP4 (W4A4) skinny linear layer on sm_100a tensor cores.
//
// Y[m][n] = g_a g_w sum_b s_a[m,b] s_w[n,b] sum_{k in b} a[m,k] w[n,k],
// M = 1..16 tokens, computed as D^T = W A^T so that the weight rows fill the
// 128-row MMA dimension and the tokens are the MMA N (= 16):
//   tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16,
//   M = 128 weight rows, N = 16 tokens, K = 64 per instruction,
//   fp32 accumulator in tensor memory, UE4M3 scales (one per 16 K) in TMEM.
//
// Work unit = one 128-row x 256-K weight tile (16 KB codes + 2 KB scales).
// The NT x KT units are cut into G = min(#SMs, units) contiguous ranges
// (stream-K split-K): every CTA streams the same number of weight bytes.
// A tile whose K range is split over several CTAs is reduced by the CTA that
// finishes it last (per-tile arrival counter); partial sums are added in
// contributor order, so results do not depend on timing.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0   TMA producer: weight tile (2-D tensor map, 128B swizzle) and
//            prepared weight scales (1-D bulk copy) for the first stages are
//            issued before griddepcontrol.wait (they never depend on the
//            previous kernel); activation tile + activation scales after it.
//   warp 1   allocates TMEM; lane 0 copies scales smem->TMEM (tcgen05.cp) and
//            issues the MMAs, releasing stages with tcgen05.commit.
//   warps 2-5 epilogue: tcgen05.ld of the 128x16 accumulator, scale by
//            g_a*g_w, optional residual, bf16 store or split-K fix-up.
#pragma once
#include "common.cuh"

namespace nvfp4sk {

constexpr int LIN_STAGES = 8;
constexpr int LIN_THREADS = 192;
constexpr uint32_t LIN_W_BYTES = 128 * 128;   // 128 rows x 256 E2M1
constexpr uint32_t LIN_A_BYTES = 16 * 128;    // 16 rows x 256 E2M1
constexpr uint32_t LIN_SF_BYTES = 2048;       // 4 x (32 x 16 B)
constexpr uint32_t LIN_STAGE_BYTES = LIN_W_BYTES + LIN_A_BYTES + 2 * LIN_SF_BYTES;   // 22528
constexpr uint32_t LIN_TX_BYTES = LIN_W_BYTES + LIN_A_BYTES + LIN_SF_BYTES;
constexpr uint32_t LIN_SMEM_BYTES = LIN_STAGES * LIN_STAGE_BYTES + 1024 + 256;
constexpr uint32_t LIN_TMEM_COLS = 128;
// TMEM column map: acc[b] at 16*b, SFA[r] at 32 + 16*r, SFB[r] at 64 + 16*r
constexpr uint32_t TM_ACC = 0, TM_SFA = 32, TM_SFB = 64;

// Instruction descriptor (kind::mxf4nvf4): A/B format E2M1 (1) in bits 7-9 and
// 10-12, K-major A and B, N>>3 in bits 17-22, scale format UE4M3 (0) in
// bit 23, M>>4 in bits 24-28, scale-factor ids 0, dense, K = 64.
constexpr uint32_t lin_idesc(uint32_t M, uint32_t N)
{
    return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (0u << 23) | ((M >> 4) << 24);
}

struct LinearParams {
    const uint8_t *w_sf;           // prepared weight scales [NT][KT][2048]
    const uint8_t *a_scales;       // [M][K/16]
    const float *g_a;
    const float *g_w;
    const __nv_bfloat16 *residual; // nullable, [M][ldy]
    __nv_bfloat16 *y;              // [M][ldy]
    float *partial;                // [G][2][16][128]
    int *counters;                 // [NT][4] (one per TMEM sub-partition)
    int64_t ldy;
    int64_t U;                     // NT * KT
    int M, N, K, NT, KT;
};

__device__ __forceinline__ int64_t lin_start(int64_t c, int64_t U, int64_t G) { return c * U / G; }
__device__ __forceinline__ int64_t lin_cta_of(int64_t u, int64_t U, int64_t G) { return ((u + 1) * G + U - 1) / U - 1; }

__global__ void __launch_bounds__(LIN_THREADS, 1)
    nvfp4_linear_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                        const LinearParams p)
{
    extern __shared__ uint8_t lin_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(lin_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + LIN_STAGES * LIN_STAGE_BYTES);
    uint64_t *empty = full + LIN_STAGES;
    uint64_t *accf = empty + LIN_STAGES;
    uint64_t *acce = accf + 2;
    uint64_t *drain = acce + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int64_t G = gridDim.x, c = blockIdx.x, U = p.U;
    const int KT = p.KT;
    const int64_t u0 = lin_start(c, U, G), u1 = lin_start(c + 1, U, G);
    const int64_t n_units = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < LIN_STAGES; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, LIN_TMEM_COLS);
        tmem_relinquish();
    }
    // zero the activation scale-factor images once; only column 0 of lines
    // 0..M-1 is rewritten per stage
    for (uint32_t i = threadIdx.x; i < LIN_STAGES * (LIN_SF_BYTES / 16); i += blockDim.x) {
        const uint32_t s = i / (LIN_SF_BYTES / 16), o = i % (LIN_SF_BYTES / 16);
        *reinterpret_cast<uint4 *>(smem + s * LIN_STAGE_BYTES + LIN_W_BYTES + LIN_A_BYTES + LIN_SF_BYTES + o * 16) =
            make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_a = policy_evict_last();
        const int64_t n_pre = n_units < LIN_STAGES ? n_units : LIN_STAGES;
        auto unit_tile = [&](int64_t i, int &t, int &kt) {
            const int64_t u = u0 + i;
            t = (int)(u / KT);
            kt = (int)(u % KT);
        };
        auto issue_w = [&](int64_t i) {
            int t, kt;
            unit_tile(i, t, kt);
            uint8_t *st = smem + (i % LIN_STAGES) * LIN_STAGE_BYTES;
            mbar_arrive_expect_tx(&full[i % LIN_STAGES], LIN_TX_BYTES);
            tma_load_2d_hint(st, &tm_w, &full[i % LIN_STAGES], kt * 128, t * 128, pol_w);
            bulk_load_hint(st + LIN_W_BYTES + LIN_A_BYTES, p.w_sf + ((int64_t)t * KT + kt) * LIN_SF_BYTES,
                           LIN_SF_BYTES, &full[i % LIN_STAGES], pol_w);
        };
        auto issue_a = [&](int64_t i) {
            int t, kt;
            unit_tile(i, t, kt);
            uint8_t *st = smem + (i % LIN_STAGES) * LIN_STAGE_BYTES;
            if (lane == 0) tma_load_2d_hint(st + LIN_W_BYTES, &tm_a, &full[i % LIN_STAGES], kt * 128, 0, pol_a);
            // activation scales: line m, column 0 of chunk j <- scales[m][kt*16 + 4j .. +3]
            const int kb = p.K / 16;
            if ((int)lane < p.M) {
                uint8_t *sfb = st + LIN_W_BYTES + LIN_A_BYTES + LIN_SF_BYTES;
                const uint8_t *src = p.a_scales + (int64_t)lane * kb;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int col = kt * 16 + 4 * j;
                    const uint32_t w = col < kb ? *reinterpret_cast<const uint32_t *>(src + col) : 0u;
                    *reinterpret_cast<uint32_t *>(sfb + j * 512 + lane * 16) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[i % LIN_STAGES]);
        };
        if (lane == 0)
            for (int64_t i = 0; i < n_pre; ++i) issue_w(i);
        pdl_wait();
        for (int64_t i = 0; i < n_pre; ++i) issue_a(i);
        int64_t issued = n_pre;
        for (int64_t i = n_pre; i < n_units; ++i) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&empty[i % LIN_STAGES], (uint32_t)(((i / LIN_STAGES) & 1) ^ 1), 101, s_abort);
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            if (lane == 0) issue_w(i);
            issue_a(i);
            issued = i + 1;
        }
        if (*s_abort && lane == 0) {
            // let every copy still in flight land before the CTA exits
            for (int64_t i = issued > LIN_STAGES ? issued - LIN_STAGES : 0; i < issued; ++i)
                mbar_wait(&full[i % LIN_STAGES], (uint32_t)((i / LIN_STAGES) & 1), 102);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = lin_idesc(128, 16);
            int64_t i = 0, seg = 0;
            bool ok = true;
            for (int64_t u = u0; u < u1 && ok; ++seg) {
                const int64_t ka = u % KT;
                const int64_t kb = (ka + (u1 - u)) < KT ? ka + (u1 - u) : KT;
                const uint32_t b = (uint32_t)(seg & 1);
                if (!mbar_wait(&acce[b], (uint32_t)(((seg >> 1) & 1) ^ 1), 103, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + TM_ACC + 16 * b;
                for (int64_t kt = ka; kt < kb; ++kt, ++i) {
                    const int s = (int)(i % LIN_STAGES);
                    if (!mbar_wait(&full[s], (uint32_t)((i / LIN_STAGES) & 1), 104, s_abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t r = (uint32_t)(i & 1);
                    const uint32_t st = smem_u32(smem + s * LIN_STAGE_BYTES);
                    const uint32_t sfa_t = tmem_base + TM_SFA + 16 * r, sfb_t = tmem_base + TM_SFB + 16 * r;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tmem_cp_32x128b_warpx4(sfa_t + 4 * j,
                                               smem_desc(st + LIN_W_BYTES + LIN_A_BYTES + 512 * j, 512, 128, SWZ_NONE));
                        tmem_cp_32x128b_warpx4(sfb_t + 4 * j,
                                               smem_desc(st + LIN_W_BYTES + LIN_A_BYTES + LIN_SF_BYTES + 512 * j, 512,
                                                         128, SWZ_NONE));
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t adesc = smem_desc(st + 32 * j, 16, 1024, SWZ_128B);
                        const uint64_t bdesc = smem_desc(st + LIN_W_BYTES + 32 * j, 16, 1024, SWZ_128B);
                        mma_mxf4nvf4(d_tmem, adesc, bdesc, idesc, sfa_t + 4 * j, sfb_t + 4 * j,
                                     (kt > ka || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(&accf[b]);
                u += kb - ka;
            }
            if (!ok) {
                // drain: wait for every MMA issued so far before TMEM is freed
                tc_commit(drain);
                mbar_wait(drain, 0, 105);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        pdl_wait();
        const uint32_t q = warp & 3;                  // TMEM sub-partition of this warp
        const int row = (int)(32 * q + lane);         // weight row within the tile
        const float gs = __fmul_rn(*p.g_a, *p.g_w);
        const int M = p.M;
        const int64_t first_tile_of_me = u0 / KT;
        int64_t seg = 0;
        for (int64_t u = u0; u < u1; ++seg) {
            const int64_t t = u / KT, ka = u % KT;
            const int64_t kb = (ka + (u1 - u)) < KT ? ka + (u1 - u) : KT;
            const uint32_t b = (uint32_t)(seg & 1);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&accf[b], (uint32_t)((seg >> 1) & 1), 106, s_abort);
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + ((32u * q) << 16) + TM_ACC + 16 * b, r);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[b]);
            const int64_t n = t * 128 + row;
            if (ka == 0 && kb == KT) {
                if (n < p.N) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        if (m < M) {
                            float o = __fmul_rn(__uint_as_float(r[m]), gs);
                            if (p.residual) o = __fadd_rn(o, __bfloat162float(p.residual[m * p.ldy + n]));
                            p.y[m * p.ldy + n] = __float2bfloat16_rn(o);
                        }
                    }
                }
            } else {
                // split-K fix-up, per warp: each warp owns rows 32q..32q+31 of the
                // tile and its own arrival counter, so no cross-warp barrier is needed
                const int slot = (t == first_tile_of_me) ? 0 : 1;
                float *P = p.partial + ((c * 2 + slot) * 16) * 128;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    if (m < M) __stcg(P + m * 128 + row, __uint_as_float(r[m]));
                __threadfence();
                __syncwarp();
                const int64_t first = lin_cta_of(t * KT, U, G), last = lin_cta_of(t * KT + KT - 1, U, G);
                int is_last = 0;
                if (lane == 0) is_last = (atomicAdd(p.counters + t * 4 + q, 1) == (int)(last - first)) ? 1 : 0;
                is_last = __shfl_sync(0xFFFFFFFFu, is_last, 0);
                if (is_last) {
                    __threadfence();
                    float acc[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc[m] = 0.f;
                    for (int64_t cc = first; cc <= last; ++cc) {
                        const int sl = ((lin_start(cc, U, G) / KT) == t) ? 0 : 1;
                        const float *Q = p.partial + ((cc * 2 + sl) * 16) * 128;
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) acc[m] = __fadd_rn(acc[m], __ldcg(Q + m * 128 + row));
                    }
                    if (n < p.N) {
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            if (m < M) {
                                float o = __fmul_rn(acc[m], gs);
                                if (p.residual) o = __fadd_rn(o, __bfloat162float(p.residual[m * p.ldy + n]));
                                p.y[m * p.ldy + n] = __float2bfloat16_rn(o);
                            }
                        }
                    }
                    if (lane == 0) p.counters[t * 4 + q] = 0;
                }
            }
            u += kb - ka;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, LIN_TMEM_COLS);
    }
}

}  // namespace nvfp4sk
