// attn.cuh -- tree-masked attention of the draft-tree nodes over the FP8
// paged KV cache on sm_100a tensor cores (flash-decoding: split over the
// context, then combine).
//
// Tree mode (the verify step): grid (splits, Hkv); one CTA = one KV head x
// one contiguous range of pages.  The 128 MMA rows are (query head w of the
// group, node i) -> row 16*w + i (rows past group*16 are zero padding), and a
// node sees the tree slots of its ancestors and itself.  Causal mode (the
// suffix prefill): grid (splits, Hq); the 128 MMA rows are up to 128 queries
// of one query head, query i at position ctx_len + i sees every position up
// to its own.  Per page of 64 tokens:
//   S = Q K^T   tcgen05.mma kind::f8f6f4, M=128, N=64, K=32 per instruction;
//               Q enters as two E4M3 terms (hi + lo) of the row-scaled bf16
//               query, K as the cached E4M3 codes (128-byte-swizzled TMA
//               tile); fp32 S in tensor memory.
//   softmax     one thread per row: S row -> registers (tcgen05.ld), ancestor
//               (or causal) mask on the pages that hold the new positions,
//               running max in the log2 domain, P' = 2^(s - m + 4) as two
//               E4M3 terms (hi + lo) stored to shared memory in the MMA's
//               core-matrix layout.  O is rescaled in tensor memory only when
//               a row max grows by more than 2^4.  Warps whose 32 rows are all
//               padding skip this work and only keep the barriers in step.
//   O += P V    M=128, N=144, K=32: the V pages are kept in HBM in the
//               core-matrix layout, so one bulk copy lands the operand; 16
//               extra operand rows (one of them all ones) make column 128 of
//               O the row sum of P', accumulated in fp32 by the tensor core.
// (Measured: an f16 P with V widened to f16 in shared memory gains nothing --
// ex2.approx.f16x2 runs at the f32 rate, 16 values per SM per clock -- and its
// operand buffers cost two of the ten ring stages, which made the last pages
// of each CTA arrive late.)
// Two softmax warpgroups take alternate pages, each with its own S and O
// accumulators in tensor memory and its own running max, so that two pages
// are in the exponent stage at once; their results are merged in the
// epilogue.
// Warp roles: 0 producer (one thread feeds a 10-stage ring: TMA K page + bulk
// V page; context pages are requested before the wait on the
// preceding kernel), 1 TMEM allocation + QK issue (one thread), 10 PV issue
// (one thread), 2-5 and 6-9 softmax.  The two issuers run independently, so
// a group's next scores never wait behind the other group's product.
// Combine: when the grid fits on the GPU at once (splits x Hkv <= #SMs, one
// CTA per SM), the CTAs of a KV head publish their split results (O / l, m,
// l per row), meet on a per-head arrival counter and each CTA then finishes
// a slice of the head's rows (fused combine, no second launch); otherwise
// tree_attn_combine_kernel merges the split results.
#pragma once
#include "common.cuh"
#include "quant.cuh"

namespace nvfp4sk {

constexpr int ATT_D = 128;
constexpr int ATT_P = 64;
constexpr int ATT_T = 16;
constexpr int ATT_ROWS = 128;
constexpr int ATT_STAGES = 10;
constexpr int ATT_THREADS = 352;
constexpr int ATT_MAX_SPLITS = 1024;
constexpr uint32_t ATT_K_BYTES = ATT_P * ATT_D;                 // 8 KB token-major page
constexpr uint32_t ATT_V_BYTES = ATT_D * ATT_P;                 // 8 KB tiled page
constexpr uint32_t ATT_ONES_BYTES = 16 * ATT_P;                 // 16 operand rows: ones, then zeros
constexpr uint32_t ATT_STAGE_BYTES = ATT_K_BYTES + ATT_V_BYTES + ATT_ONES_BYTES;   // 17 KB
constexpr uint32_t ATT_NO = ATT_D + 16;                         // O columns: 128 dims + row sum block
constexpr uint32_t ATT_PB_BYTES = ATT_ROWS * ATT_P;             // one E4M3 term of P
constexpr uint32_t ATT_OFF_P = ATT_STAGES * ATT_STAGE_BYTES;    // P[2 groups] x (hi | lo)
constexpr uint32_t ATT_OFF_X = ATT_OFF_P + 4 * ATT_PB_BYTES;    // float exchange [2][2][128]
constexpr uint32_t ATT_OFF_C = ATT_OFF_X + 2048;                // combine: bf16 rows as float [2][128]
constexpr uint32_t ATT_OFF_BAR = ATT_OFF_C + 1024;
constexpr uint32_t ATT_SMEM_BYTES = ATT_OFF_BAR + 512 + 1024;
constexpr uint32_t ATT_TMEM_COLS = 512;
constexpr uint32_t ATT_TM_S0 = 0, ATT_TM_S1 = 64;
constexpr uint32_t ATT_TM_O0 = 128, ATT_TM_O1 = 288;
constexpr uint32_t ATT_TM_Q = 448;                              // Q hi 448..479, Q lo 480..511 (A operand)
// A rescale costs a wait for the group's previous product plus a pass over O,
// and gates the whole page (the PV product waits for all four warps): with
// a threshold of 2^2, Gaussian scores, whose row max still grows by ~1.7 in
// log2 over a CTA's pages, made some row of most warps rescale on most pages.
// 2^4 leaves P' <= 2^(4 + 4) = 256 < 448 (E4M3 max) and the largest P' of a
// row >= 2^4, so a P' below the E4M3 normal range (2^-6) is < 2^-10 of it.
constexpr float ATT_TAU = 4.0f;       // log2 growth of a row max that triggers an O rescale
constexpr float ATT_PSHIFT = 4.0f;    // P' = 2^(s - m + 4) <= 2^(4 + TAU) = 256 < 448
constexpr float LOG2E = 1.4426950408889634f;
constexpr uint32_t ATT_CNT_BYTES = 256;                         // per-head arrival counters (fused combine)
static_assert(ATT_STAGE_BYTES % 1024 == 0, "K tiles need 1024-byte alignment (128-byte swizzle atoms)");
static_assert(ATT_TM_O1 + ATT_NO <= ATT_TM_Q && ATT_TM_O0 + ATT_NO <= ATT_TM_O1 && ATT_TM_Q + 64 <= ATT_TMEM_COLS,
              "tensor memory budget");
static_assert(ATT_SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Byte of (dim d, slot t) inside a V page plane: 8-dim x 16-slot core matrices
// of 128 bytes, ordered [d/8][t/16][d%8][t%16].
__host__ __device__ __forceinline__ uint32_t v_offset(uint32_t d, uint32_t t)
{
    return ((d >> 3) * (ATT_P / 16) + (t >> 4)) * 128u + (d & 7u) * 16u + (t & 15u);
}

// Instruction descriptor, kind::f8f6f4: fp32 accumulate (bits 4-5 = 1), A and
// B E4M3 (format 0), K-major, N>>3 in bits 17-22, M>>4 in bits 24-28.
constexpr uint32_t att_idesc(uint32_t M, uint32_t N) { return (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24); }

__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// same, with the A operand read from tensor memory (lane = row, 4 E4M3 per column)
__device__ __forceinline__ void mma_f8f6f4_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// packed halves: lower half <- lo, upper half <- hi
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t h)
{
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(d) : "r"(h));
    return d;
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t c)
{
    uint32_t d;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"((uint16_t)c));
    return d;
}
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four non-negative values -> E4M3 codes hi (bytes 0..3) and lo with x ~= hi + lo:
// x is rounded to f16 (11 bits), hi = E4M3(x), lo = E4M3(x - hi) (exact f16 difference).
__device__ __forceinline__ void split4_f16(float x0, float x1, float x2, float x3, uint32_t &hi, uint32_t &lo)
{
    const uint32_t a = f32x2_to_f16x2(x0, x1), b = f32x2_to_f16x2(x2, x3);
    const uint32_t ha = f16x2_to_e4m3x2(a), hb = f16x2_to_e4m3x2(b);
    const uint32_t la = f16x2_to_e4m3x2(hsub2_u32(a, e4m3x2_to_f16x2(ha)));
    const uint32_t lb = f16x2_to_e4m3x2(hsub2_u32(b, e4m3x2_to_f16x2(hb)));
    hi = ha | (hb << 16);
    lo = la | (lb << 16);
}

// x0, x1 -> (hi, lo) E4M3 pairs (byte 0 = x0, byte 1 = x1) with x ~= hi + lo, in fp32.
__device__ __forceinline__ void split2_f32(float x0, float x1, uint32_t &hi2, uint32_t &lo2)
{
    hi2 = cvt_e4m3x2(x0, x1) & 0xFFFFu;
    const uint32_t hh = e4m3x2_to_f16x2(hi2);
    const float h0 = __half2float(__ushort_as_half((unsigned short)(hh & 0xFFFFu)));
    const float h1 = __half2float(__ushort_as_half((unsigned short)(hh >> 16)));
    lo2 = cvt_e4m3x2(x0 - h0, x1 - h1) & 0xFFFFu;
}

struct AttnParams {
    const __nv_bfloat16 *q;
    int64_t ld_q;
    const uint8_t *v_pool;
    const int32_t *page_table;
    const int32_t *parent;
    const float *k_scale;
    const float *v_scale;
    float *part_o;        // [Hkv][S][group*16][128]
    float *part_ml;       // [Hkv][S][group*16][2]
    __nv_bfloat16 *out;   // [T][Hq][D]
    const float *g_act;   // static tensor scale of the fused NVFP4 output (with act)
    uint8_t *act;         // nullable: prepared NVFP4 activation of out, K = Hq*D
    int64_t ctx_len;
    int64_t n_pool_pages;
    float sm_scale;
    int *cnt;             // [grid.y] arrival counters of the fused combine (zero at call start)
    int T, Hq, Hkv, group, S, n_log_pages;
    int fuse;             // 1: fused combine in the split kernel
    int causal;           // 0: tree (grid.y = KV heads, rows 16 w + node of the group's query heads);
                          // 1: causal chain (grid.y = query heads, row = query, T <= 128)
    int rows_w;           // rows per query head in a CTA: 16 (tree) or 128 (causal)
    int nheads;           // query heads per CTA: group (tree) or 1 (causal)
};

__global__ void __launch_bounds__(ATT_THREADS, 1)
    tree_attn_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_o,
                           const AttnParams p)
{
    extern __shared__ uint8_t att_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(att_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *kv_full = reinterpret_cast<uint64_t *>(smem + ATT_OFF_BAR);
    uint64_t *kv_empty = kv_full + ATT_STAGES;
    uint64_t *s_full = kv_empty + ATT_STAGES;   // [2]
    uint64_t *s_free = s_full + 2;              // [2]
    uint64_t *p_full = s_free + 2;              // [2]
    uint64_t *p_free = p_full + 2;              // [2]
    uint64_t *q_ready = p_free + 2;
    uint64_t *o_done = q_ready + 1;
    uint64_t *drain = o_done + 1;                // [2]: QK issuer, PV issuer
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 2);
    volatile int *s_abort = reinterpret_cast<volatile int *>(tmem_holder + 1);
    volatile uint8_t *s_page_ok = reinterpret_cast<volatile uint8_t *>(tmem_holder + 2);   // [ATT_STAGES]
    float *xch = reinterpret_cast<float *>(smem + ATT_OFF_X);                             // [2][2][128]

    const int ch = blockIdx.y, split = blockIdx.x;      // CTA head: a KV head (tree) or a query head (causal)
    const int group = p.group;
    const int h = p.causal ? ch / group : ch;             // KV head
    const int hq0 = p.causal ? ch : ch * group;           // first query head of the CTA's rows
    const int rows_cta = p.nheads * p.rows_w;
    const uint32_t warp = warp_id(), lane = lane_id();
    const int pg0 = (int)((int64_t)split * p.n_log_pages / p.S);
    const int pg1 = (int)((int64_t)(split + 1) * p.n_log_pages / p.S);
    const int n_pages = pg1 - pg0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ATT_STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&p_free[b], 1);
        }
        mbar_init(q_ready, 8);
        mbar_init(o_done, 1);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, ATT_TMEM_COLS);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_k) : "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // Every role but the producer waits for the preceding kernel here (the
    // queries, the tree and the scales may be its output); the producer waits
    // only before its first tree page, see below.
    if (warp != 0) pdl_wait();
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // One converged warp; lane 0 waits and issues, in page order (stages
        // free in that order).  (Measured: one issuing thread keeps as many
        // bytes in flight as twenty; lanes that each wait on their own stage
        // diverge, and a suspended wait of one lane holds back the refills
        // of the others by microseconds.)  Page ids are read 32 at a time,
        // the next block's while the current one is issued.  Context pages of
        // the first round are requested before the wait on the preceding
        // kernel (the context and the page table are not written by it; the
        // tree slots, which the K/V append of the same step writes, are
        // loaded after it).
        auto pid_at = [&](int i) -> int32_t { return i < n_pages ? p.page_table[pg0 + i] : -1; };
        int32_t ids_cur = pid_at((int)lane), ids_nxt = pid_at(32 + (int)lane);
        int last = -1;
        bool waited = false;
        for (int i = 0; i < n_pages; ++i) {
            if (i > 0 && (i & 31) == 0) {
                ids_cur = ids_nxt;
                ids_nxt = pid_at(i + 32 + (int)lane);
            }
            const int st = i % ATT_STAGES;
            if (!waited && (i >= ATT_STAGES || (int64_t)(pg0 + i + 1) * ATT_P > p.ctx_len)) {
                pdl_wait();
                waited = true;
            }
            if (i >= ATT_STAGES) {
                bool e_ok = true;
                if (lane == 0) e_ok = mbar_wait(&kv_empty[st], (uint32_t)(((i / ATT_STAGES) - 1) & 1), 301, s_abort);
                if (!__shfl_sync(0xFFFFFFFFu, e_ok ? 1 : 0, 0)) break;
            }
            const int32_t pg = __shfl_sync(0xFFFFFFFFu, ids_cur, i & 31);
            if (lane == 0) {
                uint8_t *dst = smem + st * ATT_STAGE_BYTES;
                const bool ok = pg >= 0 && pg < p.n_pool_pages;
                s_page_ok[st] = ok ? 1 : 0;
                if (ok) {
                    mbar_arrive_expect_tx(&kv_full[st], ATT_K_BYTES + ATT_V_BYTES);
                    tma_load_2d(dst, &tm_k, &kv_full[st], 0, (int32_t)(((int64_t)pg * p.Hkv + h) * ATT_P));
                    bulk_load(dst + ATT_K_BYTES, p.v_pool + ((int64_t)pg * p.Hkv + h) * ATT_V_BYTES, ATT_V_BYTES,
                              &kv_full[st]);
                } else {
                    report_error(ERRBIT_RANGE, 302);
                    mbar_arrive(&kv_full[st]);        // page skipped: its scores are masked out
                }
            }
            last = i;
        }
        if (!waited) pdl_wait();
        // on abort, let the copies still in flight land before the CTA exits
        if (lane == 0 && *s_abort) {
            for (int i = last >= ATT_STAGES ? last - ATT_STAGES + 1 : 0; i <= last; ++i)
                mbar_wait_drain(&kv_full[i % ATT_STAGES], (uint32_t)((i / ATT_STAGES) & 1), 303);
        }
        __syncwarp();          // reconverge before the CTA-wide barrier below
    } else if (warp == 1) {
        // ------------------------------------------------------------ QK issuer
        // S = Q K^T of page i into the S buffer of group i & 1, as soon as the
        // page has landed and the group has read that buffer's previous page
        if (lane == 0) {
            constexpr uint32_t idesc_s = att_idesc(128, ATT_P);
            const uint32_t q_hi = tmem_base + ATT_TM_Q, q_lo = q_hi + 32u;
            bool ok = mbar_wait(q_ready, 0, 310, s_abort);
            for (int i = 0; i < n_pages && ok; ++i) {
                const int st = i % ATT_STAGES, g = i & 1;
                if (!mbar_wait(&kv_full[st], (uint32_t)((i / ATT_STAGES) & 1), 312, s_abort)) { ok = false; break; }
                if (i >= 2 && !mbar_wait(&s_free[g], (uint32_t)(((i - 2) >> 1) & 1), 313, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t k_s = smem_u32(smem + st * ATT_STAGE_BYTES);
                const uint32_t s_t = tmem_base + (g ? ATT_TM_S1 : ATT_TM_S0);
#pragma unroll
                for (int t = 0; t < ATT_D / 32; ++t) {
                    const uint64_t kd = smem_desc(k_s + 32 * t, 16, 1024, SWZ_128B);
                    mma_f8f6f4_ta(s_t, q_hi + 8u * t, kd, idesc_s, t > 0 ? 1u : 0u);
                    mma_f8f6f4_ta(s_t, q_lo + 8u * t, kd, idesc_s, 1u);
                }
                tc_commit(&s_full[g]);
            }
            // every QK product is complete before tensor memory is released
            tc_commit(&drain[0]);
            mbar_wait_drain(&drain[0], 0, 314);
        }
        __syncwarp();
    } else if (warp == 10) {
        // ------------------------------------------------------------ PV issuer
        // O_g += P V of page j once group g has written P (hi, lo) for it
        if (lane == 0) {
            constexpr uint32_t idesc_o = att_idesc(128, ATT_NO);
            bool o_init[2] = {false, false};
            bool ok = true;
            for (int j = 0; j < n_pages && ok; ++j) {
                const int g = j & 1;
                if (!mbar_wait(&p_full[g], (uint32_t)((j >> 1) & 1), 311, s_abort)) { ok = false; break; }
                tc_fence_after();
                if (s_page_ok[j % ATT_STAGES]) {
                    const uint32_t v_s = smem_u32(smem + (j % ATT_STAGES) * ATT_STAGE_BYTES + ATT_K_BYTES);
                    const uint32_t p_hi = smem_u32(smem + ATT_OFF_P + g * 2 * ATT_PB_BYTES), p_lo = p_hi + ATT_PB_BYTES;
                    const uint32_t o_t = tmem_base + (g ? ATT_TM_O1 : ATT_TM_O0);
#pragma unroll
                    for (int t = 0; t < ATT_P / 32; ++t) {
                        const uint64_t vd = smem_desc(v_s + 256 * t, 128, 512, SWZ_NONE);
                        mma_f8f6f4(o_t, smem_desc(p_hi + 256 * t, 128, 512, SWZ_NONE), vd, idesc_o,
                                   (o_init[g] || t > 0) ? 1u : 0u);
                        mma_f8f6f4(o_t, smem_desc(p_lo + 256 * t, 128, 512, SWZ_NONE), vd, idesc_o, 1u);
                    }
                    o_init[g] = true;
                }
                tc_commit(&p_free[g]);
                tc_commit(&kv_empty[j % ATT_STAGES]);
            }
            if (ok) {
                tc_commit(o_done);
            } else {
                tc_commit(&drain[1]);
                mbar_wait_drain(&drain[1], 0, 315);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax groups
        const int g = (int)(warp - 2) >> 2;                   // 0: even pages, 1: odd pages
        const int gt = (int)threadIdx.x - 64 - 128 * g;       // thread index within the group
        const uint32_t qd = warp & 3;                         // TMEM sub-partition
        const int r = (int)(32 * qd + lane);                  // MMA row
        const int w = r / p.rows_w, node = r % p.rows_w;      // query head within the CTA, node / query
        const bool row_ok = w < p.nheads;
        const int hq = hq0 + w;
        const int T = p.T;
        const int64_t L = p.ctx_len;
        const uint32_t row_t = tmem_base + ((32u * qd) << 16);
        const uint32_t s_t = row_t + (g ? ATT_TM_S1 : ATT_TM_S0);
        const uint32_t o_t = row_t + (g ? ATT_TM_O1 : ATT_TM_O0);
        uint8_t *pb = smem + ATT_OFF_P + g * 2 * ATT_PB_BYTES;
        // a warp whose 32 rows are all padding does no softmax work (the
        // products of its rows are never read) and only keeps the barriers in step
        const bool pad_warp = !__any_sync(0xFFFFFFFFu, row_ok && node < p.T);

        // ---- Q -> two E4M3 terms, row scaled by a power of two into [128, 256);
        //      group g converts dims 64g .. 64g+63 of row r.  Every global
        //      load of the prologue is issued first, in one round trip.
        float c_row;
        uint32_t anc = 0;
        int32_t pid = -1, pid_next = -1;
        {
            const bool has_q = row_ok && node < T;
            const int par_l = (!p.causal && (int)lane < T) ? p.parent[lane] : -1;
            const float k_sc = p.k_scale[h];
            if (g < n_pages) pid = p.page_table[pg0 + g];
            if (g + 2 < n_pages) pid_next = p.page_table[pg0 + g + 2];
            uint4 qraw[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                qraw[k] = has_q ? *reinterpret_cast<const uint4 *>(p.q + node * p.ld_q + (int64_t)hq * ATT_D + 64 * g + 8 * k)
                                : make_uint4(0, 0, 0, 0);
            float amax = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t wd[4] = {qraw[k].x, qraw[k].y, qraw[k].z, qraw[k].w};
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(wd[j] << 16)),
                                             fabsf(__uint_as_float(wd[j] & 0xFFFF0000u))));
            }
            xch[g * 128 + r] = amax;
            // the ones block of every stage: operand row 128 (16 bytes per 16-token chunk) = 1.0, rest 0
            for (int idx = (int)threadIdx.x - 64; idx < ATT_STAGES * (int)(ATT_ONES_BYTES / 16); idx += 256) {
                const uint32_t off = (uint32_t)(idx % (ATT_ONES_BYTES / 16)) * 16u;
                const uint32_t v = (off < 512u && (off & 127u) == 0u) ? 0x38383838u : 0u;
                *reinterpret_cast<uint4 *>(smem + (idx / (ATT_ONES_BYTES / 16)) * ATT_STAGE_BYTES + ATT_K_BYTES +
                                           ATT_V_BYTES + off) = make_uint4(v, v, v, v);
            }
            named_bar_sync(1, 256);
            amax = fmaxf(xch[r], xch[128 + r]);
            int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 : 0;
            e = max(-120, min(127, e));
            const float qs = amax > 0.f ? __uint_as_float((uint32_t)(127 + 7 - e) << 23) : 1.f;
            c_row = __fdiv_rn(k_sc * p.sm_scale * LOG2E, qs);
            // A operand of S = Q K^T in tensor memory: row r in lane r, dims 4c .. 4c+3
            // in column c; this group writes columns 16g .. 16g+15 of each term
            uint32_t hw[16], lw[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {                      // dims 64g + 8k .. 64g + 8k + 7
                const uint32_t wv[4] = {qraw[k].x, qraw[k].y, qraw[k].z, qraw[k].w};
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t h01, l01, h23, l23;
                    split2_f32(__uint_as_float(wv[2 * j] << 16) * qs, __uint_as_float(wv[2 * j] & 0xFFFF0000u) * qs,
                               h01, l01);
                    split2_f32(__uint_as_float(wv[2 * j + 1] << 16) * qs,
                               __uint_as_float(wv[2 * j + 1] & 0xFFFF0000u) * qs, h23, l23);
                    hw[2 * k + j] = h01 | (h23 << 16);
                    lw[2 * k + j] = l01 | (l23 << 16);
                }
            }
            tmem_st_x16(row_t + ATT_TM_Q + 16u * (uint32_t)g, hw);
            tmem_st_x16(row_t + ATT_TM_Q + 32u + 16u * (uint32_t)g, lw);
            tmem_wait_st();
            // ancestors (and self) of every node by pointer doubling: lane t holds
            // node t's set and a jump pointer; each round joins the set of the
            // node the pointer names and doubles the pointer's reach, so
            // log2(ATT_T) rounds cover any chain of ATT_T nodes
            if (!p.causal) {
                int jmp = par_l;
                const bool bad = (int)lane < T && jmp >= T;  // malformed tree: parent id out of range
                if (bad || jmp < 0) jmp = -1;
                uint32_t set = (int)lane < T ? 1u << lane : 0u;
#pragma unroll
                for (int k = 0; (1 << k) < ATT_T; ++k) {
                    const int src = jmp >= 0 ? jmp : (int)lane;
                    const uint32_t set2 = __shfl_sync(0xFFFFFFFFu, set, src);
                    const int jmp2 = __shfl_sync(0xFFFFFFFFu, jmp, src);
                    if (jmp >= 0) {
                        set |= set2;
                        jmp = jmp2;
                    }
                }
                anc = __shfl_sync(0xFFFFFFFFu, set, has_q ? node : 0);
                if (!has_q) anc = 0;
                if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) report_error(ERRBIT_RANGE, 305);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }

        float m_ref = -INFINITY;
        bool ok = true;
        for (int i = g; i < n_pages; i += 2) {
            const bool vpage = pid >= 0 && pid < p.n_pool_pages;
            pid = pid_next;
            if (i + 4 < n_pages) pid_next = p.page_table[pg0 + i + 4];
            bool w_ok = true;
            if (lane == 0) w_ok = mbar_wait(&s_full[g], (uint32_t)((i >> 1) & 1), 320, s_abort);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0)) { ok = false; break; }
            tc_fence_after();
            uint32_t s[64];
            {
                uint32_t (&s0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&s[0]);
                uint32_t (&s1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&s[32]);
                tmem_ld_x32(s_t, s0);
                tmem_ld_x32(s_t + 32u, s1);
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[g]);
            if (!vpage) {                                      // no product for this page
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[g]);
                continue;
            }
            const int64_t pos0 = (int64_t)(pg0 + i) * ATT_P;
            bool waited = false;
            if (!pad_warp) {
                if (pos0 + ATT_P > L) {
                    // column j holds new-position slot t0 + j (negative: context);
                    // bit j of vis = column j visible to this row
                    const int t0 = (int)(pos0 - L);            // > -64
                    uint64_t vis;
                    if (p.causal) {                            // slots 0 .. node (node < T)
                        const int lim = min(node, T - 1) - t0;
                        vis = lim >= 63 ? ~0ull : lim < 0 ? 0ull : ((2ull << lim) - 1ull);
                    } else {                                   // context, then the ancestor slots
                        const uint64_t ctx = t0 >= 0 ? 0ull : ((1ull << (-t0)) - 1ull);
                        vis = ctx | (t0 >= 0 ? ((uint64_t)anc >> t0) : ((uint64_t)anc << (-t0)));
                    }
                    const uint32_t v_lo = (uint32_t)vis, v_hi = (uint32_t)(vis >> 32);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (!((v_lo >> j) & 1u)) s[j] = 0xFF800000u;          // -inf
                        if (!((v_hi >> j) & 1u)) s[32 + j] = 0xFF800000u;
                    }
                }
                // row max as a tree (8 independent chains, then 3 levels): a
                // 63-deep chain of dependent maxes is on every page's critical path
                float m8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) m8[k] = __uint_as_float(s[k]);
#pragma unroll
                for (int j = 8; j < 64; ++j) m8[j & 7] = fmaxf(m8[j & 7], __uint_as_float(s[j]));
                const float mr = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                const float mx = mr * c_row;
                const bool need = mx > m_ref + ATT_TAU;
                const bool resc = need && m_ref > -INFINITY;
                if (__any_sync(0xFFFFFFFFu, resc)) {
                    // every product of this group so far must be in O before it is rescaled
                    bool r_ok = true;
                    if (lane == 0) r_ok = mbar_wait(&p_free[g], (uint32_t)(((i - 2) >> 1) & 1), 321, s_abort);
                    if (!__shfl_sync(0xFFFFFFFFu, r_ok ? 1 : 0, 0)) { ok = false; break; }
                    waited = true;
                    tc_fence_after();
                    const float alpha = resc ? fast_exp2(m_ref - mx) : 1.f;
#pragma unroll 1
                    for (uint32_t col = 0; col < ATT_NO; col += 16) {
                        uint32_t o[16];
                        tmem_ld_32x32b_x16(o_t + col, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tmem_st_x16(o_t + col, o);
                    }
                    tmem_wait_st();
                }
                if (need) m_ref = mx;
            }
            uint32_t ph[16], pl[16];
            if (!pad_warp) {
                const float nb = m_ref > -INFINITY ? ATT_PSHIFT - m_ref : 0.f;
#pragma unroll
                for (int j = 0; j < 64; j += 4)
                    split4_f16(fast_exp2(fmaf(__uint_as_float(s[j]), c_row, nb)),
                               fast_exp2(fmaf(__uint_as_float(s[j + 1]), c_row, nb)),
                               fast_exp2(fmaf(__uint_as_float(s[j + 2]), c_row, nb)),
                               fast_exp2(fmaf(__uint_as_float(s[j + 3]), c_row, nb)), ph[j >> 2], pl[j >> 2]);
            }
            if (pos0 + ATT_P > L + T) {
                // slots past the last written position may hold any byte (NaN codes
                // included); zero their V (this thread: dimension r) so 0 * V stays 0
                const bool k_ok = mbar_wait(&kv_full[i % ATT_STAGES], (uint32_t)((i / ATT_STAGES) & 1), 324, s_abort);
                if (!__all_sync(0xFFFFFFFFu, k_ok)) { ok = false; break; }
                // slots tz .. 63 of dimension r: 16 contiguous bytes per 16-slot chunk
                uint8_t *vd = smem + (i % ATT_STAGES) * ATT_STAGE_BYTES + ATT_K_BYTES + v_offset((uint32_t)r, 0);
                const int tz = (int)(L + T - pos0);           // 1 .. 63: the last page holds position L+T-1
                int c = tz >> 4;
                if (tz & 15) {
                    for (int t = tz & 15; t < 16; ++t) vd[c * 128 + t] = 0;
                    ++c;
                }
                for (; c < ATT_P / 16; ++c) *reinterpret_cast<uint4 *>(vd + c * 128) = make_uint4(0, 0, 0, 0);
            }
            // the P buffer of this group's previous page must have been consumed
            if (!waited && i >= 2) {
                bool f_ok = true;
                if (lane == 0) f_ok = mbar_wait(&p_free[g], (uint32_t)(((i - 2) >> 1) & 1), 322, s_abort);
                if (!__shfl_sync(0xFFFFFFFFu, f_ok ? 1 : 0, 0)) { ok = false; break; }
            }
            if (!pad_warp) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {                  // tokens 16c .. 16c+15
                    const uint32_t off = (((uint32_t)r >> 3) * 4u + (uint32_t)c) * 128u + ((uint32_t)r & 7u) * 16u;
                    *reinterpret_cast<uint4 *>(pb + off) = make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
                    *reinterpret_cast<uint4 *>(pb + ATT_PB_BYTES + off) =
                        make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[g]);
        }

        // ---- merge the two groups' (m, O) and write the split result:
        //      o = O / l (V code units), m, l; group g writes dims 64g .. 64g+63
        bool d_ok = ok && n_pages > 0;
        if (d_ok && lane == 0) d_ok = mbar_wait(o_done, 0, 323, s_abort);
        d_ok = __shfl_sync(0xFFFFFFFFu, d_ok ? 1 : 0, 0) != 0;
        xch[256 + g * 128 + r] = m_ref;
        named_bar_sync(1, 256);
        const float mA = xch[256 + r], mB = xch[384 + r];
        const int64_t prow = ((int64_t)ch * p.S + split) * rows_cta + r;
        if (d_ok) {
            tc_fence_after();
            const float M = fmaxf(mA, mB);
            const float wA = mA > -INFINITY ? fast_exp2(mA - M) : 0.f;
            const float wB = mB > -INFINITY ? fast_exp2(mB - M) : 0.f;
            const float lA = __uint_as_float(tmem_ld_x1(row_t + ATT_TM_O0 + 128u));
            const float lB = __uint_as_float(tmem_ld_x1(row_t + ATT_TM_O1 + 128u));
            tmem_wait_ld();
            const float l = (wA > 0.f ? wA * lA : 0.f) + (wB > 0.f ? wB * lB : 0.f);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float ca = wA > 0.f ? wA * inv : 0.f, cb = wB > 0.f ? wB * inv : 0.f;
            float *dst = p.part_o + prow * ATT_D;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t col = 64u * (uint32_t)g + 32u * cc;
                uint32_t oa[32], ob[32];
                tmem_ld_x32(row_t + ATT_TM_O0 + col, oa);
                tmem_ld_x32(row_t + ATT_TM_O1 + col, ob);
                tmem_wait_ld();
                // without the fused combine: dims col .. col+31 of the CTA's rows
                // form box 2g+cc of the tensor store below, staged in the ring
                // (free after o_done) as 128-byte rows, 16-byte chunk j of row r
                // at chunk j ^ (r % 8)
                uint8_t *box = smem + (2u * (uint32_t)g + (uint32_t)cc) * (uint32_t)rows_cta * 128u + (uint32_t)r * 128u;
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float v[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float a = ca > 0.f ? ca * __uint_as_float(oa[j + k]) : 0.f;
                            const float b = cb > 0.f ? cb * __uint_as_float(ob[j + k]) : 0.f;
                            v[k] = a + b;
                        }
                        if (p.fuse)
                            __stcg(reinterpret_cast<float4 *>(dst + col + j), make_float4(v[0], v[1], v[2], v[3]));
                        else
                            *reinterpret_cast<float4 *>(box + ((((uint32_t)j >> 2) ^ ((uint32_t)r & 7u)) << 4)) =
                                make_float4(v[0], v[1], v[2], v[3]);
                    }
                }
            }
            if (row_ok && g == 0) __stcg(reinterpret_cast<float2 *>(p.part_ml + prow * 2), make_float2(M - ATT_PSHIFT, l));
        } else if (n_pages == 0 && row_ok && g == 0) {
            __stcg(reinterpret_cast<float2 *>(p.part_ml + prow * 2), make_float2(0.f, 0.f));
        }
        if (!p.fuse) {
            // four TMA tensor stores (32 dims x rows_cta rows each) of the staged
            // split result; the store is complete before the CTA exits
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 64 && n_pages > 0 && !*s_abort) {
                const int32_t row0 = (int32_t)(((int64_t)ch * p.S + split) * rows_cta);
#pragma unroll
                for (int b = 0; b < 4; ++b) tma_store_2d(&tm_o, smem + b * rows_cta * 128, 128 * b, row0);
                bulk_commit();
                bulk_wait<0>();
            }
        }

        if (p.fuse) {
            // ---- fused combine: publish, meet the head's other splits, then
            //      merge rows r0 .. r1-1 of this KV head (row = w*T + node).
            //      The barrier orders every thread's partial stores before the
            //      one release-add (a release is cumulative over what its thread
            //      has synchronised with); likewise the acquiring poll, then the
            //      barrier, before any thread reads the other splits' results.
            named_bar_sync(1, 256);
            if (threadIdx.x == 64) {
                red_release_gpu_add(p.cnt + ch, 1);
                const bool all_in = poll_counter_ge(p.cnt + ch, p.S, 325, s_abort);
                if (!all_in) *s_abort = 1;
                xch[0] = (all_in && !*s_abort) ? 1.f : 0.f;        // one decision for every thread
            }
            named_bar_sync(1, 256);
            const bool merge = xch[0] != 0.f;
            const int nr = p.nheads * T;
            const int r0 = (int)((int64_t)split * nr / p.S), r1 = (int)((int64_t)(split + 1) * nr / p.S);
            const int nrow = r1 - r0;
            // warps = R row slots x Q split slices: rows go in parallel when the
            // CTA has many (causal mode), splits when it has few (tree mode)
            const int sw = (int)warp - 2;                          // softmax warp 0..7
            const int R = nrow < 8 ? (nrow > 0 ? nrow : 1) : 8, Q = 8 / R;
            const int rs = sw % R, qs = sw / R;
            const bool worker = qs < Q;
            float *accs = reinterpret_cast<float *>(smem + ATT_OFF_P);   // [8 warps][128], the idle P buffer
            float *crow = reinterpret_cast<float *>(smem + ATT_OFF_C) + 128 * g;
            const float vsc = p.v_scale[h];
            for (int k0 = 0; merge && k0 < nrow; k0 += R) {
                const int j = k0 + rs;                             // this warp's row of the round
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                if (worker && j < nrow) {
                    const int row = r0 + j, ww = row / T, nd = row % T;
                    const int64_t base = (int64_t)ch * p.S * rows_cta + ww * p.rows_w + nd;   // + s * rows_cta
                    // one round trip: the (m, l) of every split (lane holds splits
                    // lane, lane+32, ...) and this warp's partial rows (splits qs,
                    // qs+Q, ..., up to 24 per lane) are requested together
                    float2 ml[5];
                    float4 v[24];
#pragma unroll
                    for (int i = 0; i < 5; ++i) {
                        const int sp = (int)lane + 32 * i;
                        ml[i] = sp < p.S ? __ldcg(reinterpret_cast<const float2 *>(p.part_ml + 2 * (base + sp * rows_cta)))
                                         : make_float2(0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < 24; ++k) {
                        const int sp = qs + k * Q;
                        v[k] = sp < p.S ? __ldcg(reinterpret_cast<const float4 *>(p.part_o + (base + sp * rows_cta) * ATT_D) + lane)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    float mloc = -INFINITY;
#pragma unroll
                    for (int i = 0; i < 5; ++i)
                        if (ml[i].y > 0.f) mloc = fmaxf(mloc, ml[i].x);
                    const float M = warp_max(mloc);
                    float wv[5], dloc = 0.f;
#pragma unroll
                    for (int i = 0; i < 5; ++i) {
                        wv[i] = ml[i].y > 0.f ? ml[i].y * fast_exp2(ml[i].x - M) : 0.f;
                        dloc += wv[i];
                    }
                    const float den = warp_sum(dloc);
                    const float inv = den > 0.f ? 1.f / den : 0.f;
                    auto weight = [&](int sp) {                        // sp warp-uniform
                        float wsel = wv[0];
#pragma unroll
                        for (int i = 1; i < 5; ++i)
                            if ((sp >> 5) == i) wsel = wv[i];
                        return __shfl_sync(0xFFFFFFFFu, wsel, sp & 31) * inv;
                    };
#pragma unroll
                    for (int k = 0; k < 24; ++k) {
                        const int sp = qs + k * Q;
                        if (sp < p.S) {
                            const float w = weight(sp);
                            acc.x += w * v[k].x; acc.y += w * v[k].y; acc.z += w * v[k].z; acc.w += w * v[k].w;
                        }
                    }
                    // splits beyond the first 24 of this warp (many splits, few rows)
                    for (int sp = qs + 24 * Q; sp < p.S; sp += Q) {
                        const float4 x = __ldcg(reinterpret_cast<const float4 *>(p.part_o + (base + sp * rows_cta) * ATT_D) + lane);
                        const float w = weight(sp);
                        acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
                    }
                }
                reinterpret_cast<float4 *>(accs + 128 * sw)[lane] = acc;
                named_bar_sync(1, 256);
                // outputs of the round's rows: group g takes row slots g, g+2, ...
                for (int rr = g; rr < R && k0 + rr < nrow; rr += 2) {
                    const int row = r0 + k0 + rr, ww = row / T, nd = row % T;
                    const int d = gt;
                    float o = 0.f;
                    for (int qq = 0; qq < Q; ++qq) o += accs[128 * (qq * R + rr) + d];
                    const __nv_bfloat16 obf = __float2bfloat16_rn(o * vsc);
                    const int hq2 = hq0 + ww;
                    p.out[((int64_t)nd * p.Hq + hq2) * ATT_D + d] = obf;
                    if (p.act) {
                        crow[d] = __bfloat162float(obf);
                        named_bar_sync(2 + g, 128);
                        if (d < ATT_D / 16) {
                            float v[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k) v[k] = crow[16 * d + k];
                            uint2 pk;
                            const uint32_t sc = quant_block16(v, *p.g_act, pk);
                            store_prepared(p.act, nd, (int64_t)hq2 * (ATT_D / 16) + d, pk, sc);
                        }
                        named_bar_sync(2 + g, 128);
                    }
                }
                named_bar_sync(1, 256);                            // accs reused by the next round
            }
            // the last CTA of the head through here resets its counter for the next call
            named_bar_sync(1, 256);
            if (threadIdx.x == 64 && merge) {
                if (atomicAdd(p.cnt + ch, 1) == 2 * p.S - 1) atomicExch(p.cnt + ch, 0);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, ATT_TMEM_COLS);
    }
}

// out[i][hq][:] = sum_s w_s o_s / sum_s w_s * v_scale[h],  w_s = l_s 2^(m_s - M).
// One CTA per (node, query head), 4 warps: warp j sums splits j, j+4, ... for
// all 128 dims (4 per lane); the partial rows of its first 16 splits are
// requested before the weights are known, so the kernel waits on about one
// round of L2 loads.  Warp sums are added in warp order (deterministic).
constexpr int CMB_PF = 16;
__global__ void __launch_bounds__(ATT_D) tree_attn_combine_kernel(const AttnParams p)
{
    __shared__ float w_s[ATT_MAX_SPLITS];
    __shared__ float l_s[ATT_MAX_SPLITS];
    __shared__ float red[ATT_D / 32];
    __shared__ float4 xs[4][ATT_D / 4];
    pdl_wait();
    pdl_launch_dependents();
    const int i = blockIdx.x, hq = blockIdx.y, tid = threadIdx.x;
    const int wp = tid >> 5, lane = tid & 31;
    const int h = hq / p.group;                                   // KV head
    const int ch = p.causal ? hq : h, w = p.causal ? 0 : hq % p.group;
    const int S = p.S;
    const int64_t rows_cta = (int64_t)p.nheads * p.rows_w;
    auto row = [&](int s) { return ((int64_t)ch * S + s) * rows_cta + (int64_t)w * p.rows_w + i; };
    // the scales the tail needs go out with the split results, not after
    // the reductions (two round trips off the end of the call)
    const float vsc = p.v_scale[h];
    const float g_act = p.act ? *p.g_act : 0.f;
    float4 pv[CMB_PF];
#pragma unroll
    for (int k = 0; k < CMB_PF; ++k) {
        const int s = wp + 4 * k;
        pv[k] = s < S ? __ldcg(reinterpret_cast<const float4 *>(p.part_o + row(s) * ATT_D) + lane)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mloc = -INFINITY;
    for (int s = tid; s < S; s += ATT_D) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + 2 * row(s)));
        w_s[s] = ml.y > 0.f ? ml.x : -INFINITY;
        l_s[s] = ml.y;
        if (ml.y > 0.f) mloc = fmaxf(mloc, ml.x);
    }
    mloc = warp_max(mloc);
    if (lane == 0) red[wp] = mloc;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float dloc = 0.f;
    for (int s = tid; s < S; s += ATT_D) {
        const float m = w_s[s];
        const float ws = m > -INFINITY ? l_s[s] * fast_exp2(m - M) : 0.f;
        w_s[s] = ws;
        dloc += ws;
    }
    dloc = warp_sum(dloc);
    if (lane == 0) red[wp] = dloc;
    __syncthreads();
    const float den = (red[0] + red[1]) + (red[2] + red[3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < CMB_PF; ++k) {
        const int s = wp + 4 * k;
        const float ws = s < S ? w_s[s] : 0.f;
        if (ws > 0.f) {
            acc.x += ws * pv[k].x; acc.y += ws * pv[k].y; acc.z += ws * pv[k].z; acc.w += ws * pv[k].w;
        }
    }
    for (int s = wp + 4 * CMB_PF; s < S; s += 4) {
        const float ws = w_s[s];
        if (ws > 0.f) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.part_o + row(s) * ATT_D) + lane);
            acc.x += ws * v.x; acc.y += ws * v.y; acc.z += ws * v.z; acc.w += ws * v.w;
        }
    }
    xs[wp][lane] = acc;
    __syncthreads();
    const float *xf = reinterpret_cast<const float *>(xs);
    const float num = (xf[tid] + xf[ATT_D + tid]) + (xf[2 * ATT_D + tid] + xf[3 * ATT_D + tid]);
    const float o = den > 0.f ? num / den * vsc : 0.f;
    const __nv_bfloat16 ob = __float2bfloat16_rn(o);
    p.out[((int64_t)i * p.Hq + hq) * ATT_D + tid] = ob;
    if (p.act) {
        // NVFP4 of the bf16 output row with the static tensor scale: the 8 blocks of
        // 16 dims of this head are blocks hq*8 .. hq*8+7 of row i (K = Hq*D)
        __shared__ float orow[ATT_D];
        orow[tid] = __bfloat162float(ob);
        __syncthreads();
        if (tid < ATT_D / 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = orow[16 * tid + k];
            uint2 pk;
            const uint32_t sc = quant_block16(v, g_act, pk);
            store_prepared(p.act, i, (int64_t)hq * (ATT_D / 16) + tid, pk, sc);
        }
    }
}

}  // namespace nvfp4sk
