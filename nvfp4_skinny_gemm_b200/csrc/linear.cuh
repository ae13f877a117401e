// linear.cuh -- NVFP4 (W4A4) skinny linear layer on sm_100a tensor cores.
//
// Y[m][n] = g_a g_w sum_b s_a[m,b] s_w[n,b] sum_{k in b} a[m,k] w[n,k],
// M = 1..16 tokens, computed as D^T = W A^T so that the weight rows fill the
// 128-row MMA dimension and the tokens are the MMA N (= 16):
//   tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16,
//   M = 128 weight rows, N = 16 tokens, K = 64 per instruction,
//   fp32 accumulator in tensor memory, UE4M3 scales (one per 16 K) in TMEM.
//
// Operands arrive pre-tiled in exactly the shared-memory image the MMA reads
// (128-byte swizzled E2M1 rows, scale factors as the 32 x 16-byte blocks that
// tcgen05.cp replicates into tensor memory):
//   weight unit (tile t of 128 rows, chunk c of 512 K):  36 KB contiguous
//     [2 x 16 KB codes (one per 256-K swizzle atom) | 8 x 512 B scale images]
//   activation chunk c: 8 KB contiguous
//     [2 x 2 KB codes (16 rows) | 8 x 512 B scale images]
// so one pipeline stage is two bulk copies (cp.async.bulk) and nothing else.
// (A single issuing thread sustains ~7 TB/s over the GPU with >= 32 KB
// requests; small per-tile requests and generic shared-memory writes were
// what limited the earlier 2-D tensor-map version to ~3.4 TB/s.)
//
// Work unit = one weight unit.  The NT x KC units are cut into
// G = min(#SMs, units) contiguous ranges (stream-K split-K), so every CTA
// streams the same number of weight bytes.  A tile whose K range is split
// over several CTAs is reduced by its owner, the CTA holding its first K
// chunk (which reaches that tile last): the other contributors publish fp32
// partial sums and bump a per-tile, per-sub-partition arrival counter; the
// owner polls the counter and loads their partials while its own products
// are still in flight, then adds them in contributor order, so results do
// not depend on timing.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0   producer: weight units of the first stages are requested before
//            griddepcontrol.wait (weights never depend on the previous
//            kernel); activation chunks after it.
//   warp 1   allocates TMEM; lane 0 issues the MMAs, releasing stages with
//            tcgen05.commit.
//   warps 2-5 stage the scale factors of every unit into tensor memory with
//            tcgen05.st (one warp per TMEM sub-partition), a few units ahead of
//            the MMAs; and the epilogue: tcgen05.ld of the 128x16 accumulator,
//            scale by g_a*g_w, optional residual, bf16 store or split-K fix-up.
// (Measured on B200: a tcgen05.cp of one scale block takes ~47 cycles of the
// tensor pipe and an N = 16 block-scaled MMA ~52, and the two serialise: the
// 16 copies + 8 MMAs of a unit held the pipe ~1,165 cycles, 70% of the
// unit's HBM time.  Staging the scales through the idle epilogue warps leaves
// only the MMAs on the pipe.)
#pragma once
#include "common.cuh"

namespace nvfp4sk {

constexpr int LIN_STAGES = 4;
constexpr int LIN_THREADS = 192;
constexpr int LIN_PF = 7;                         // split-K partials prefetched by a tile's owner
constexpr int LIN_KC = 512;                       // K elements per unit / chunk
constexpr int LIN_KSTEPS = LIN_KC / 64;           // MMA steps per unit
constexpr uint32_t LIN_W_ATOM = 128 * 128;        // 128 rows x 256 E2M1, swizzled
constexpr uint32_t LIN_A_ATOM = 16 * 128;         // 16 rows x 256 E2M1, swizzled
constexpr uint32_t LIN_SF_IMG = 512;              // 32 lines x 16 B
constexpr uint32_t LIN_W_UNIT = 2 * LIN_W_ATOM + LIN_KSTEPS * LIN_SF_IMG;    // 36864
constexpr uint32_t LIN_A_UNIT = 2 * LIN_A_ATOM + LIN_KSTEPS * LIN_SF_IMG;    // 8192
constexpr uint32_t LIN_STAGE_BYTES = LIN_W_UNIT + LIN_A_UNIT;                // 45056 = 44 * 1024
constexpr uint32_t LIN_OFF_BAR = LIN_STAGES * LIN_STAGE_BYTES;
constexpr uint32_t LIN_SMEM_BYTES = LIN_OFF_BAR + 256 + 1024;
// gate+up with SwiGLU: two stages of (gate unit, up unit, activation chunk),
// then per epilogue warp a 16 x 33 float transpose buffer
constexpr uint32_t LIN_SW_X_BYTES = 4 * 16 * 33 * 4;
constexpr uint32_t LIN_SMEM_BYTES_SW = 2 * (2 * LIN_W_UNIT + LIN_A_UNIT) + 256 + LIN_SW_X_BYTES + 1024;
static_assert(LIN_SMEM_BYTES_SW <= 227 * 1024, "shared memory budget");
constexpr uint32_t LIN_TMEM_COLS = 512;
constexpr int LIN_NACC = 1;                       // independent accumulators per tile (MMA j -> j % LIN_NACC)
constexpr int LIN_SFB_SLOTS = 11;                 // activation-scale chunks kept resident in TMEM
// TMEM columns: accumulator a of buffer b at 16*(LIN_NACC*b + a) (16 fp32
// columns = 16 tokens; the MMAs of a tile rotate over the LIN_NACC
// accumulators so that consecutive products do not wait on each other, and
// the epilogue adds them in a fixed order); the weight scales SFA and the
// activation scales SFB of the unit in pipeline stage s, 32 columns each per
// stage (4 per MMA step), or, when the activation scales stay resident, up to
// LIN_SFB_SLOTS K chunks of SFB in place of the per-stage SFB buffers.
// Scale-factor column addresses handed to the MMA stay multiples of 4.
constexpr uint32_t TM_ACC = 0, TM_SFA = 32 * LIN_NACC, TM_SFB = TM_SFA + 32 * LIN_STAGES, TM_SFB_RES = TM_SFB;
static_assert(TM_SFB + 32 * LIN_STAGES <= LIN_TMEM_COLS && TM_SFB_RES + 32 * LIN_SFB_SLOTS <= LIN_TMEM_COLS,
              "tensor memory budget");

// Instruction descriptor (kind::mxf4nvf4): A/B format E2M1 (1) in bits 7-9 and
// 10-12, K-major A and B, N>>3 in bits 17-22, scale format UE4M3 (0) in
// bit 23, M>>4 in bits 24-28, scale-factor ids 0, dense, K = 64.
constexpr uint32_t lin_idesc(uint32_t M, uint32_t N)
{
    return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (0u << 23) | ((M >> 4) << 24);
}

struct LinearParams {
    const uint8_t *w;              // prepared weight units [NT][KC][36864]
    const uint8_t *a;              // prepared activation chunks [KC][8192]
    const float *g_a;
    const float *g_w;
    const __nv_bfloat16 *residual; // nullable, [M][ldy]
    __nv_bfloat16 *y;              // [M][ldy]
    float *partial;                // [G][2][128 rows][16 tokens]
    int *counters;                 // [NT][4] (one per TMEM sub-partition)
    int64_t ldy;
    int64_t U;                     // NT * KC (gate+up with SwiGLU: gate tiles x KC)
    int M, N, NT, KC;              // (gate+up with SwiGLU: N = F features, NT = F / 128)
    uint8_t *sw_act;               // gate+up with SwiGLU: prepared NVFP4 activation [M] x F
    const float *sw_g;             //   and its static tensor scale
};

// defined in quant.cuh (the SwiGLU epilogue quantises like the SwiGLU quantiser)
__device__ __forceinline__ uint32_t quant_block16(const float (&v)[16], float g, uint2 &packed);
__device__ __forceinline__ void store_prepared(uint8_t *act, int64_t r, int64_t blk, uint2 pk, uint32_t sc);
__device__ __forceinline__ float swiglu_bf16(float gate, float up);

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wait (bounded) until *p == want; returns false and records a timeout otherwise.
__device__ __forceinline__ bool poll_counter(const int *p, int want, uint32_t site, volatile int *abort)
{
    if (ld_acquire_gpu(p) == want) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 8; ++i)
            if (ld_acquire_gpu(p) == want) return true;
        if (abort && *abort) return false;
        if (globaltimer() - t0 > g_timeout_ns) {
            report_error(ERRBIT_TIMEOUT, site);
            if (abort) *abort = 1;
            return false;
        }
    }
}

// Wait (bounded) until *p >= want; returns false and records a timeout otherwise.
// Polls with a short sleep in between: many CTAs may wait on one counter, and
// back-to-back polls of one L2 line slow the memory traffic of the CTAs that
// are still working.
__device__ __forceinline__ bool poll_counter_ge(const int *p, int want, uint32_t site, volatile int *abort)
{
    if (ld_acquire_gpu(p) >= want) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        __nanosleep(64);
        for (int i = 0; i < 2; ++i)
            if (ld_acquire_gpu(p) >= want) return true;
        if (abort && *abort) return false;
        if (globaltimer() - t0 > g_timeout_ns) {
            report_error(ERRBIT_TIMEOUT, site);
            if (abort) *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ int64_t lin_start(int64_t c, int64_t U, int64_t G) { return c * U / G; }
__device__ __forceinline__ int64_t lin_cta_of(int64_t u, int64_t U, int64_t G) { return ((u + 1) * G + U - 1) / U - 1; }

// The activation scales of K chunk kc are the same for every weight tile:
// when a CTA sweeps all K chunks at least four times (an LM-head-like shape:
// many tiles, short K), each chunk's scales are staged into tensor memory
// once (slot kc - kc0 mod KC) and reused by every later tile.
// (Not with SwiGLU: its TMEM columns past the per-stage scales are taken.)
template <bool SW>
__device__ __forceinline__ bool lin_sfb_resident(int64_t n_units, int64_t KC)
{
    return !SW && n_units >= 4 * KC && KC <= LIN_SFB_SLOTS;
}

template <bool SW>
__global__ void __launch_bounds__(LIN_THREADS, 1)
    nvfp4_linear_kernel(const LinearParams p)
{
    // SW (gate+up with SwiGLU): a unit is the gate unit u and the up unit
    // U + u of the same K chunk (the up rows follow the gate rows in the
    // weight), two accumulators per tile, two stages of 80 KB.
    constexpr int NH = SW ? 2 : 1;                        // weight units per stage
    constexpr int STG = SW ? 2 : LIN_STAGES;
    constexpr uint32_t STB = NH * LIN_W_UNIT + LIN_A_UNIT;
    constexpr uint32_t OFF_BAR = STG * STB;
    constexpr int PF = SW ? 2 : LIN_PF;
    constexpr int PW = 16 * NH;                           // partial-sum floats per row
    constexpr uint32_t T_SFA = TM_ACC + 2 * 16 * NH;      // after 2 buffers x NH accumulators
    constexpr uint32_t T_SFB = T_SFA + 32 * NH * STG;
    static_assert(LIN_NACC == 1, "one accumulator per tile and half");
    static_assert(T_SFB + 32 * STG <= LIN_TMEM_COLS, "tensor memory budget");
    static_assert(!SW || OFF_BAR + 256 + LIN_SW_X_BYTES + 1024 <= LIN_SMEM_BYTES_SW, "shared memory budget");
    extern __shared__ uint8_t lin_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(lin_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *empty = full + STG;
    uint64_t *accf = empty + STG;
    uint64_t *acce = accf + 2;
    uint64_t *drain = acce + 2;
    uint64_t *sf_ready = drain + 1;                 // [STG]: scales of the stage's unit are in TMEM
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(sf_ready + STG);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int64_t G = gridDim.x, c = blockIdx.x, U = p.U;
    const int KC = p.KC;
    const int64_t u0 = lin_start(c, U, G), u1 = lin_start(c + 1, U, G);
    const int64_t n_units = u1 - u0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(&full[s], 2);          // weight-unit arrive.expect_tx + activation arrive.expect_tx
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4);
        }
        mbar_init(drain, 1);
        for (int st = 0; st < STG; ++st) mbar_init(&sf_ready[st], 4);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, LIN_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            const int64_t n_pre = n_units < STG ? n_units : STG;
            auto issue_w = [&](int64_t i) {
                const int s = (int)(i % STG);
                mbar_arrive_expect_tx(&full[s], NH * LIN_W_UNIT);
                bulk_load_hint(smem + s * STB, p.w + (u0 + i) * (int64_t)LIN_W_UNIT, LIN_W_UNIT, &full[s], pol_w);
                if (SW)
                    bulk_load_hint(smem + s * STB + LIN_W_UNIT, p.w + (U + u0 + i) * (int64_t)LIN_W_UNIT, LIN_W_UNIT,
                                   &full[s], pol_w);
            };
            auto issue_a = [&](int64_t i) {
                const int s = (int)(i % STG);
                const int64_t kc = (u0 + i) % KC;
                mbar_arrive_expect_tx(&full[s], LIN_A_UNIT);
                bulk_load_hint(smem + s * STB + NH * LIN_W_UNIT, p.a + kc * (int64_t)LIN_A_UNIT, LIN_A_UNIT, &full[s],
                               pol_a);
            };
            for (int64_t i = 0; i < n_pre; ++i) issue_w(i);
            pdl_wait();
            for (int64_t i = 0; i < n_pre; ++i) issue_a(i);
            int64_t issued = n_pre;
            for (int64_t i = n_pre; i < n_units; ++i) {
                if (!mbar_wait(&empty[i % STG], (uint32_t)(((i / STG) & 1) ^ 1), 101, s_abort)) break;
                issue_w(i);
                issue_a(i);
                issued = i + 1;
            }
            if (*s_abort) {
                // let every copy still in flight land before the CTA exits
                for (int64_t i = issued > STG ? issued - STG : 0; i < issued; ++i)
                    mbar_wait_drain(&full[i % STG], (uint32_t)((i / STG) & 1), 102);
            }
        } else {
            pdl_wait();
        }
        __syncwarp();          // reconverge before the CTA-wide barrier below
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = lin_idesc(128, 16);
            int64_t i = 0, seg = 0;
            bool ok = true;
            const bool sfb_resident = lin_sfb_resident<SW>(n_units, KC);
            const int64_t kc0 = u0 % KC;
            for (int64_t u = u0; u < u1 && ok; ++seg) {
                const int64_t ka = u % KC;
                const int64_t kend = (ka + (u1 - u)) < KC ? ka + (u1 - u) : KC;
                const uint32_t b = (uint32_t)(seg & 1);
                if (!mbar_wait(&acce[b], (uint32_t)(((seg >> 1) & 1) ^ 1), 103, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + TM_ACC + 16 * NH * b;
                for (int64_t kc = ka; kc < kend; ++kc, ++i) {
                    const int s = (int)(i % STG);
                    const uint32_t par = (uint32_t)((i / STG) & 1);
                    if (!mbar_wait(&full[s], par, 104, s_abort) || !mbar_wait(&sf_ready[s], par, 109, s_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w_s = smem_u32(smem + s * STB);
                    const uint32_t a_s = w_s + NH * LIN_W_UNIT;
                    const uint32_t sfb_t = sfb_resident ? tmem_base + TM_SFB_RES + 32 * (uint32_t)((kc - kc0 + KC) % KC)
                                                        : tmem_base + T_SFB + 32 * (uint32_t)s;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const uint32_t sfa_t = tmem_base + T_SFA + 32 * (uint32_t)(NH * s + h);
#pragma unroll
                        for (int j = 0; j < LIN_KSTEPS; ++j) {
                            const uint32_t atom = (uint32_t)(j >> 2), ko = 32u * (uint32_t)(j & 3);
                            const uint64_t adesc =
                                smem_desc(w_s + h * LIN_W_UNIT + atom * LIN_W_ATOM + ko, 16, 1024, SWZ_128B);
                            const uint64_t bdesc = smem_desc(a_s + atom * LIN_A_ATOM + ko, 16, 1024, SWZ_128B);
                            mma_mxf4nvf4(d_tmem + 16 * h, adesc, bdesc, idesc, sfa_t + 4 * j, sfb_t + 4 * j,
                                         (kc > ka || j > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty[s]);
                }
                if (!ok) break;
                tc_commit(&accf[b]);
                u += kend - ka;
            }
            if (!ok) {
                // drain: wait for every MMA issued so far before TMEM is freed
                tc_commit(drain);
                mbar_wait_drain(drain, 0, 105);
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
        const int64_t first_tile_of_me = u0 / KC;
        // Scale staging: the weight and activation scale images of unit i (each
        // 8 blocks of 32 lines x 16 bytes, line l = rows l, l+32, l+64, l+96)
        // go to every TMEM sub-partition (this warp writes its own), the layout
        // the block-scaled MMA reads; then one arrive on sf_ready of the stage.
        // The per-stage buffers of unit i are free again once unit i has landed:
        // the producer refilled its stage only after the MMAs of unit i-STAGES
        // had completed.
        const bool sfb_resident = lin_sfb_resident<SW>(n_units, KC);
        const int64_t kc0 = u0 % KC;
        const uint32_t lane_base = tmem_base + ((32u * q) << 16);
        uint32_t sfb_loaded = 0;
        int64_t next_sf = 0;
        bool sf_ok = true;
        auto stage_scales = [&](int64_t i) -> bool {
            const int s = (int)(i % STG);
            const bool landed = mbar_wait(&full[s], (uint32_t)((i / STG) & 1), 108, s_abort);
            if (!__all_sync(0xFFFFFFFFu, landed)) return false;
            const uint8_t *st = smem + s * STB;
            uint32_t v[32];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
#pragma unroll
                for (int j = 0; j < LIN_KSTEPS; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(st + h * LIN_W_UNIT + 2 * LIN_W_ATOM +
                                                                     LIN_SF_IMG * j + 16 * lane);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st_x32(lane_base + T_SFA + 32 * (uint32_t)(NH * s + h), v);
            }
            uint32_t sfb_col = T_SFB + 32 * (uint32_t)s;
            bool copy_sfb = true;
            if (sfb_resident) {
                const uint32_t slot = (uint32_t)((((u0 + i) % KC) - kc0 + KC) % KC);
                sfb_col = TM_SFB_RES + 32 * slot;
                copy_sfb = !((sfb_loaded >> slot) & 1u);
                sfb_loaded |= 1u << slot;
            }
            if (copy_sfb) {
#pragma unroll
                for (int j = 0; j < LIN_KSTEPS; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(st + NH * LIN_W_UNIT + 2 * LIN_A_ATOM +
                                                                     LIN_SF_IMG * j + 16 * lane);
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                tmem_st_x32(lane_base + sfb_col, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sf_ready[s]);
            return true;
        };
        auto stage_scales_until = [&](int64_t last) {
            while (sf_ok && next_sf <= last && next_sf < n_units) sf_ok = stage_scales(next_sf++);
            return sf_ok;
        };
        int64_t seg = 0;
        for (int64_t u = u0; u < u1; ++seg) {
            const int64_t t = u / KC, ka = u % KC;
            const int64_t kend = (ka + (u1 - u)) < KC ? ka + (u1 - u) : KC;
            const uint32_t b = (uint32_t)(seg & 1);
            // stage the scales of this tile's units and of up to STAGES-1 later
            // ones, so that the MMAs keep going while this tile is written out
            if (!stage_scales_until((u - u0) + (kend - ka) - 1 + (STG - 1))) break;
            const bool whole = ka == 0 && kend == KC;
            const int64_t first = whole ? c : lin_cta_of(t * KC, U, G);
            const int64_t last = whole ? c : lin_cta_of(t * KC + KC - 1, U, G);
            // Split tile: the CTA holding its first K chunk owns it.  That chunk
            // range ends the owner's own range, so the owner reaches this tile
            // last; it polls the other contributors' arrivals and loads their
            // partial sums while its own products are still in flight, then adds
            // them to its accumulator in contributor order.
            const bool owner = !whole && c == first;
            float part[PF][PW];
            bool ok = true;
            if (owner) {
                // lane 0's acquire, then the warp barrier (which orders memory
                // among the warp's threads), before any lane reads a partial sum
                if (lane == 0) ok = poll_counter(p.counters + t * 4 + q, (int)(last - first), 107, s_abort);
                __syncwarp();
                ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
#pragma unroll
                for (int k = 0; k < PF; ++k) {
                    const int64_t cc = first + 1 + k;
                    if (cc <= last) {
                        const int sl = ((lin_start(cc, U, G) / KC) == t) ? 0 : 1;
                        const float4 *Q = reinterpret_cast<const float4 *>(p.partial + ((cc * 2 + sl) * 128 + row) * PW);
#pragma unroll
                        for (int v = 0; v < PW / 4; ++v) {
                            const float4 f = __ldcg(Q + v);
                            part[k][4 * v] = f.x; part[k][4 * v + 1] = f.y; part[k][4 * v + 2] = f.z; part[k][4 * v + 3] = f.w;
                        }
                    }
                }
            }
            if (lane == 0) ok = mbar_wait(&accf[b], (uint32_t)((seg >> 1) & 1), 106, s_abort);
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            uint32_t r[PW];                               // [half][token]
            {
                const uint32_t acc_t = tmem_base + ((32u * q) << 16) + TM_ACC + 16 * NH * b;
                tmem_ld_32x32b_x16(acc_t, *reinterpret_cast<uint32_t (*)[16]>(&r[0]));
                if constexpr (SW) tmem_ld_32x32b_x16(acc_t + 16, *reinterpret_cast<uint32_t (*)[16]>(&r[16]));
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[b]);
            const int64_t n = t * 128 + row;
            if (whole || owner) {
                float acc[PW];
#pragma unroll
                for (int m = 0; m < PW; ++m) acc[m] = __uint_as_float(r[m]);
                if (owner) {
#pragma unroll
                    for (int k = 0; k < PF; ++k)
                        if (first + 1 + k <= last) {
#pragma unroll
                            for (int m = 0; m < PW; ++m) acc[m] = __fadd_rn(acc[m], part[k][m]);
                        }
                    // tiles split over more than PF + 1 CTAs: the rest, in order
                    for (int64_t cc = first + 1 + PF; cc <= last; ++cc) {
                        const int sl = ((lin_start(cc, U, G) / KC) == t) ? 0 : 1;
                        const float4 *Q = reinterpret_cast<const float4 *>(p.partial + ((cc * 2 + sl) * 128 + row) * PW);
#pragma unroll
                        for (int v = 0; v < PW / 4; ++v) {
                            const float4 f = __ldcg(Q + v);
                            acc[4 * v] = __fadd_rn(acc[4 * v], f.x);
                            acc[4 * v + 1] = __fadd_rn(acc[4 * v + 1], f.y);
                            acc[4 * v + 2] = __fadd_rn(acc[4 * v + 2], f.z);
                            acc[4 * v + 3] = __fadd_rn(acc[4 * v + 3], f.w);
                        }
                    }
                    if (lane == 0) p.counters[t * 4 + q] = 0;
                }
                if constexpr (SW) {
                    // gate and up of feature n for the 16 tokens, rounded to bf16 as a
                    // stored linear output would be, then SwiGLU rounded to bf16 (the
                    // arithmetic of the SwiGLU quantiser); a per-warp transpose through
                    // shared memory gives each lane one NVFP4 block (token, 16 features)
                    float *xs = reinterpret_cast<float *>(smem + OFF_BAR + 256) + q * (16 * 33);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float gt = __bfloat162float(__float2bfloat16_rn(__fmul_rn(acc[m], gs)));
                        const float up = __bfloat162float(__float2bfloat16_rn(__fmul_rn(acc[16 + m], gs)));
                        xs[m * 33 + lane] = swiglu_bf16(gt, up);
                    }
                    __syncwarp();
                    const int tok = (int)(lane & 15u), hb = (int)(lane >> 4);
                    float v[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) v[k] = xs[tok * 33 + 16 * hb + k];
                    __syncwarp();
                    if (tok < M) {
                        uint2 pk;
                        const uint32_t sc = quant_block16(v, *p.sw_g, pk);
                        store_prepared(p.sw_act, tok, (t * 128 + 32 * q + 16 * hb) / 16, pk, sc);
                    }
                } else if (n < p.N) {
                    // y may alias the residual (y = h + linear(h)): every residual
                    // load goes out before the first store
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc[m] = __fmul_rn(acc[m], gs);
                    if (p.residual) {
                        __nv_bfloat16 res[16];
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            res[m] = m < M ? p.residual[m * p.ldy + n] : __float2bfloat16_rn(0.f);
#pragma unroll
                        for (int m = 0; m < 16; ++m) acc[m] = __fadd_rn(acc[m], __bfloat162float(res[m]));
                    }
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m < M) p.y[m * p.ldy + n] = __float2bfloat16_rn(acc[m]);
                }
            } else {
                // contributor: publish the partial sum, then one release add on the
                // tile's arrival counter (per warp: each warp owns rows 32q..32q+31)
                const int slot = (t == first_tile_of_me) ? 0 : 1;
                float4 *P = reinterpret_cast<float4 *>(p.partial + ((c * 2 + slot) * 128 + row) * PW);
#pragma unroll
                for (int v = 0; v < PW / 4; ++v)
                    __stcg(P + v, make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                              __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                // the warp barrier orders every lane's stores before lane 0's
                // release add (a release is cumulative over what its thread has
                // synchronised with), so no separate fence is needed
                __syncwarp();
                if (lane == 0) red_release_gpu_add(p.counters + t * 4 + q, 1);
            }
            u += kend - ka;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, LIN_TMEM_COLS);
    }
}

// ---- operand preparation ----------------------------------------------------
// Offset, inside a 128-byte-swizzled image (rows of 128 B, base 1024-aligned),
// of byte b of row r: the 16-byte chunk index is XORed with r % 8 (the layout
// a 128-byte-swizzle TMA load would produce and the MMA descriptor expects).
__host__ __device__ __forceinline__ uint32_t swz128(uint32_t r, uint32_t b)
{
    return r * 128u + ((((b >> 4) ^ (r & 7u)) << 4) | (b & 15u));
}

// Weight units: for tile t, chunk c:
//   atom a, row r, byte b   <- codes[t*128 + r][c*256 + a*128 + b]
//   scale image j, line l, byte 4*cc + kb <- scales[t*128 + l + 32*cc][c*32 + 4*j + kb]
// zero outside the matrix.  One CTA per unit; each thread writes whole
// 16-byte chunks: the 128-byte swizzle permutes whole 16-byte chunks of a
// code row, so a code chunk is one 16-byte source load, and a scale chunk
// gathers four 4-byte pieces (rows l, l+32, l+64, l+96).  Needs codes
// 16-byte and scales 4-byte aligned (checked by the caller).
__global__ void __launch_bounds__(256) prepare_weight_kernel(const uint8_t *__restrict__ codes,
                                                             const uint8_t *__restrict__ scales, int64_t N, int64_t K,
                                                             int64_t KC, uint8_t *__restrict__ out)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t unit = blockIdx.x;
    const int64_t t = unit / KC, c = unit % KC;
    const int64_t kbytes = K / 2, kb = K / 16;
    uint8_t *u = out + unit * (int64_t)LIN_W_UNIT;
#pragma unroll
    for (int k = threadIdx.x; k < (int)(LIN_W_UNIT / 16); k += 256) {             // 9 chunks per thread, all in flight
        uint4 v = make_uint4(0, 0, 0, 0);
        if (k < (int)(2 * LIN_W_ATOM / 16)) {
            const int a = k >> 10, r = (k >> 3) & 127, j = k & 7;       // atom, row, stored chunk
            const int64_t row = t * 128 + r;
            const int64_t col = c * 256 + a * 128 + (int64_t)((j ^ (r & 7)) << 4);
            if (row < N && col < kbytes) v = *reinterpret_cast<const uint4 *>(codes + row * kbytes + col);
        } else {
            const int k2 = k - (int)(2 * LIN_W_ATOM / 16), jimg = k2 >> 5, l = k2 & 31;
            const int64_t blk = c * 32 + 4 * jimg;
            uint32_t w[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int64_t row = t * 128 + l + 32 * cc;
                w[cc] = (row < N && blk < kb) ? *reinterpret_cast<const uint32_t *>(scales + row * kb + blk) : 0u;
            }
            v = make_uint4(w[0], w[1], w[2], w[3]);
        }
        *reinterpret_cast<uint4 *>(u + 16 * (int64_t)k) = v;
    }
}

}  // namespace nvfp4sk
