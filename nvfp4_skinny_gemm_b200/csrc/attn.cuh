// attn.cuh -- tree-masked attention of the draft-tree nodes over the FP8
// paged KV cache (flash-decoding: split over the context, then combine).
//
// Grid (splits, Hkv); one CTA = one KV head x one contiguous range of pages.
// Warps 0..group-1 each own one query head of the group and all 16 nodes
// (16 MMA rows); the last warp is the producer: per page it loads the K page
// (8 KB, 2-D TMA with 128-byte swizzle) and the V page (8 KB, 1-D bulk copy,
// stored dimension-major) into a ring of shared-memory stages.
//
// Both contractions run on FP8 tensor-core MMAs (mma.sync m16n8k32 e4m3,
// fp32 accumulate), reading the cached E4M3 codes straight from shared
// memory; the per-head K/V scales are applied to scores / outputs instead.
// The bf16 query (scaled per row by a power of two) and the probabilities
// (scaled by 256) are each written as a sum of two E4M3 terms hi + lo, so
// each contraction is two MMAs and the operands keep ~8 significant bits.
// Token and dimension orders inside a page are permuted (consistently for
// Q, K, P and V) so that every fragment is one conflict-free 16-byte load.
// Softmax is online in the log2 domain; rows are reduced with quad shuffles.
#pragma once
#include "common.cuh"

namespace nvfp4sk {

constexpr int ATT_D = 128;
constexpr int ATT_P = 64;
constexpr int ATT_T = 16;
constexpr int ATT_STAGES = 4;
constexpr uint32_t ATT_K_BYTES = ATT_P * ATT_D;     // 8 KB, token-major
constexpr uint32_t ATT_V_BYTES = ATT_D * ATT_P;     // 8 KB, dimension-major
constexpr uint32_t ATT_STAGE_BYTES = ATT_K_BYTES + ATT_V_BYTES;
constexpr uint32_t ATT_SMEM_BYTES = ATT_STAGES * ATT_STAGE_BYTES + 1024 + 256;
constexpr float LOG2E = 1.4426950408889634f;

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
    int64_t ctx_len;
    int64_t n_pool_pages;
    float sm_scale;
    int T, Hq, Hkv, group, S, n_log_pages;
};

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// x -> (hi, lo) E4M3 codes with x ~= value(hi) + value(lo)
__device__ __forceinline__ void split_e4m3(float x, uint32_t &hi, uint32_t &lo)
{
    hi = cvt_e4m3x2(x, 0.f) & 0xFFu;
    const float r = x - e4m3_to_float(hi);
    lo = cvt_e4m3x2(r, 0.f) & 0xFFu;
}

// two floats -> two (hi, lo) pairs packed into bytes [0..1] of hi2 / lo2
__device__ __forceinline__ void split_e4m3x2(float x0, float x1, uint32_t &hi2, uint32_t &lo2, float &sum)
{
    const uint32_t h = cvt_e4m3x2(x0, x1);          // byte0 = x0, byte1 = x1
    uint32_t hh;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"((uint16_t)h));
    const float h0 = __half2float(__ushort_as_half((unsigned short)(hh & 0xFFFFu)));
    const float h1 = __half2float(__ushort_as_half((unsigned short)(hh >> 16)));
    const float r0 = x0 - h0, r1 = x1 - h1;
    const uint32_t l = cvt_e4m3x2(r0, r1);
    uint32_t ll;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(ll) : "h"((uint16_t)l));
    sum += (h0 + h1) + (__half2float(__ushort_as_half((unsigned short)(ll & 0xFFFFu))) +
                        __half2float(__ushort_as_half((unsigned short)(ll >> 16))));
    hi2 = h & 0xFFFFu;
    lo2 = l & 0xFFFFu;
}

__global__ void __launch_bounds__(8 * 32, 1)
    tree_attn_split_kernel(const __grid_constant__ CUtensorMap tm_k, const AttnParams p)
{
    extern __shared__ uint8_t att_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(att_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ATT_STAGES * ATT_STAGE_BYTES);
    uint64_t *empty = full + ATT_STAGES;
    volatile int *s_valid = reinterpret_cast<volatile int *>(empty + ATT_STAGES);
    volatile int *s_abort = s_valid + ATT_STAGES;

    const int h = blockIdx.y, split = blockIdx.x;
    const int group = p.group;
    const uint32_t warp = warp_id(), lane = lane_id();
    const int pg0 = (int)((int64_t)split * p.n_log_pages / p.S);
    const int pg1 = (int)((int64_t)(split + 1) * p.n_log_pages / p.S);
    const int n_pages = pg1 - pg0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ATT_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], group);
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    if ((int)warp == group) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int i = 0; i < n_pages; ++i) {
                const int st = i % ATT_STAGES;
                if (i >= ATT_STAGES &&
                    !mbar_wait(&empty[st], (uint32_t)(((i / ATT_STAGES) & 1) ^ 1), 301, s_abort))
                    break;
                const int32_t pg = p.page_table[pg0 + i];
                const bool valid = pg >= 0 && pg < p.n_pool_pages;
                s_valid[st] = valid ? 1 : 0;
                uint8_t *dst = smem + st * ATT_STAGE_BYTES;
                if (valid) {
                    mbar_arrive_expect_tx(&full[st], ATT_STAGE_BYTES);
                    tma_load_2d(dst, &tm_k, &full[st], 0, (int32_t)(((int64_t)pg * p.Hkv + h) * ATT_P));
                    bulk_load(dst + ATT_K_BYTES, p.v_pool + ((int64_t)pg * p.Hkv + h) * ATT_V_BYTES, ATT_V_BYTES,
                              &full[st]);
                } else {
                    report_error(ERRBIT_RANGE, 302);
                    mbar_arrive(&full[st]);
                }
            }
            if (*s_abort) {
                for (int i = n_pages > ATT_STAGES ? n_pages - ATT_STAGES : 0; i < n_pages; ++i)
                    mbar_wait(&full[i % ATT_STAGES], (uint32_t)((i / ATT_STAGES) & 1), 303);
            }
        }
        return;
    }
    if ((int)warp > group) return;

    // ---------------------------------------------------------------- compute
    const int hq = h * group + (int)warp;
    const int g = (int)(lane >> 2), c = (int)(lane & 3);
    const int T = p.T;
    const int64_t L = p.ctx_len;

    // query fragments: rows g (node g) and g+8 (node g+8), dims 32c..32c+31
    float qv[2][32];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int node = g + 8 * rr;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (node < T) w = *reinterpret_cast<const uint4 *>(p.q + node * p.ld_q + (int64_t)hq * ATT_D + 32 * c + 8 * i);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                qv[rr][8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
                qv[rr][8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
            }
        }
    }
    float c_row[2];
    uint32_t anc[2];
    uint32_t qa_hi[4][4], qa_lo[4][4];   // [k-step][reg]
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        float amax = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(qv[rr][k]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        // power-of-two row scale 2^(7 - floor(log2 amax)) puts the row max in [128, 256)
        int e = 0;
        if (amax > 0.f) e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
        e = max(-100, min(100, e));
        const float qs = amax > 0.f ? __uint_as_float((uint32_t)(127 + 7 - e) << 23) : 1.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) qv[rr][k] *= qs;
        c_row[rr] = __fdiv_rn(p.k_scale[h] * p.sm_scale * LOG2E, qs);
        // ancestor mask of node g + 8 rr
        uint32_t m = 0;
        const int node = g + 8 * rr;
        if (node < T) {
            int a = node;
            for (int it = 0; it < ATT_T && a >= 0; ++it) {
                if (a >= T) {                      // malformed tree: parent id out of range
                    report_error(ERRBIT_RANGE, 305);
                    break;
                }
                m |= 1u << a;
                a = p.parent[a];
            }
        }
        anc[rr] = m;
    }
    // dims of k-step t = 2u + v: a0/b0 <-> 32c + 16u + 8v + 0..3, a2/b1 <-> +4..7
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int base = 16 * (t >> 1) + 8 * (t & 1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                uint32_t hw = 0, lw = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t hb, lb;
                    split_e4m3(qv[rr][base + 4 * half + j], hb, lb);
                    hw |= hb << (8 * j);
                    lw |= lb << (8 * j);
                }
                qa_hi[t][2 * half + rr] = hw;   // reg order: a0 (g,lo-k) a1 (g+8,lo-k) a2 (g,hi-k) a3 (g+8,hi-k)
                qa_lo[t][2 * half + rr] = lw;
            }
        }
    }

    float O[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) O[nd][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    for (int i = 0; i < n_pages; ++i) {
        const int st = i % ATT_STAGES;
        if (!mbar_wait(&full[st], (uint32_t)((i / ATT_STAGES) & 1), 304, s_abort)) break;
        if (s_valid[st]) {
            const uint8_t *kt = smem + st * ATT_STAGE_BYTES;
            const uint8_t *vt = kt + ATT_K_BYTES;
            const int64_t pos0 = (int64_t)(pg0 + i) * ATT_P;
            float sacc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            // k-steps outermost so that consecutive MMAs update different n-tiles
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                uint4 kw[8];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int tok = 16 * (g >> 1) + 8 * (nt >> 2) + 4 * ((nt & 3) >> 1) + 2 * (nt & 1) + (g & 1);
                    kw[nt] = *reinterpret_cast<const uint4 *>(kt + tok * 128 + (((2 * c + u) ^ (tok & 7)) << 4));
                }
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mma_e4m3_16832(sacc[nt], qa_hi[2 * u], kw[nt].x, kw[nt].y);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mma_e4m3_16832(sacc[nt], qa_hi[2 * u + 1], kw[nt].z, kw[nt].w);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mma_e4m3_16832(sacc[nt], qa_lo[2 * u], kw[nt].x, kw[nt].y);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mma_e4m3_16832(sacc[nt], qa_lo[2 * u + 1], kw[nt].z, kw[nt].w);
            }
            // scale, mask, row max
            const bool tail = pos0 + ATT_P > L;
            float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int rr = e >> 1;
                    float s2 = sacc[nt][e] * c_row[rr];
                    if (tail) {
                        const int tok = 16 * c + 8 * (nt >> 2) + 4 * ((nt & 3) >> 1) + 2 * (nt & 1) + (e & 1);
                        const int64_t pos = pos0 + tok;
                        bool vis = pos < L;
                        if (!vis) {
                            const int64_t j = pos - L;
                            vis = j < T && ((anc[rr] >> j) & 1u);
                        }
                        if (!vis) s2 = -INFINITY;
                    }
                    sacc[nt][e] = s2;
                    tmax[rr] = fmaxf(tmax[rr], s2);
                }
            }
            float alpha[2], muse[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xFFFFFFFFu, tmax[rr], 1));
                tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xFFFFFFFFu, tmax[rr], 2));
                const float mn = fmaxf(m_run[rr], tmax[rr]);
                muse[rr] = mn == -INFINITY ? 0.f : mn;
                alpha[rr] = fast_exp2(m_run[rr] - muse[rr]);
                m_run[rr] = mn;
            }
            // probabilities x 256 as (hi, lo) E4M3 pairs, packed into PV A fragments
            uint32_t pa_hi[2][4], pa_lo[2][4];
            float psum[2] = {0.f, 0.f};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {          // a0/a1 (n-tiles 4w,4w+1) a2/a3 (4w+2,4w+3)
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int nA = 4 * w + 2 * half, nB = nA + 1;
                        const float x0 = fast_exp2(sacc[nA][2 * rr] - muse[rr]) * 256.f;
                        const float x1 = fast_exp2(sacc[nA][2 * rr + 1] - muse[rr]) * 256.f;
                        const float x2 = fast_exp2(sacc[nB][2 * rr] - muse[rr]) * 256.f;
                        const float x3 = fast_exp2(sacc[nB][2 * rr + 1] - muse[rr]) * 256.f;
                        uint32_t h01, l01, h23, l23;
                        split_e4m3x2(x0, x1, h01, l01, psum[rr]);
                        split_e4m3x2(x2, x3, h23, l23, psum[rr]);
                        pa_hi[w][2 * half + rr] = h01 | (h23 << 16);
                        pa_lo[w][2 * half + rr] = l01 | (l23 << 16);
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) l_run[rr] = l_run[rr] * alpha[rr] + psum[rr];
            // four dimension tiles at a time: their MMAs are independent
#pragma unroll
            for (int nd0 = 0; nd0 < 16; nd0 += 4) {
                uint4 x[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int nd = nd0 + k;
                    O[nd][0] *= alpha[0]; O[nd][1] *= alpha[0];
                    O[nd][2] *= alpha[1]; O[nd][3] *= alpha[1];
                    x[k] = *reinterpret_cast<const uint4 *>(vt + (8 * nd + g) * ATT_P + 16 * c);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_e4m3_16832(O[nd0 + k], pa_hi[0], x[k].x, x[k].y);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_e4m3_16832(O[nd0 + k], pa_hi[1], x[k].z, x[k].w);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_e4m3_16832(O[nd0 + k], pa_lo[0], x[k].x, x[k].y);
#pragma unroll
                for (int k = 0; k < 4; ++k) mma_e4m3_16832(O[nd0 + k], pa_lo[1], x[k].z, x[k].w);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }

    // partial result of this split: o = O / l (V code units), m, l
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        l_run[rr] += __shfl_xor_sync(0xFFFFFFFFu, l_run[rr], 1);
        l_run[rr] += __shfl_xor_sync(0xFFFFFFFFu, l_run[rr], 2);
    }
    const int64_t rowbase = (((int64_t)h * p.S + split) * group + warp) * 16;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int node = g + 8 * rr;
        const float inv = l_run[rr] > 0.f ? 1.f / l_run[rr] : 0.f;
        float *dst = p.part_o + (rowbase + node) * ATT_D;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd)
            __stcg(reinterpret_cast<float2 *>(dst + 8 * nd + 2 * c),
                   make_float2(O[nd][2 * rr] * inv, O[nd][2 * rr + 1] * inv));
        if (c == 0) __stcg(reinterpret_cast<float2 *>(p.part_ml + (rowbase + node) * 2), make_float2(m_run[rr], l_run[rr]));
    }
}

// out[i][hq][:] = sum_s w_s o_s / sum_s w_s * v_scale[h],  w_s = l_s 2^(m_s - M)
__global__ void __launch_bounds__(ATT_D) tree_attn_combine_kernel(const AttnParams p)
{
    pdl_wait();
    pdl_launch_dependents();
    const int i = blockIdx.x, hq = blockIdx.y, d = threadIdx.x;
    const int h = hq / p.group, w = hq % p.group;
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) {
        const int64_t r = (((int64_t)h * p.S + s) * p.group + w) * 16 + i;
        M = fmaxf(M, __ldcg(p.part_ml + 2 * r));
    }
    float num = 0.f, den = 0.f;
    for (int s = 0; s < p.S; ++s) {
        const int64_t r = (((int64_t)h * p.S + s) * p.group + w) * 16 + i;
        const float m = __ldcg(p.part_ml + 2 * r), l = __ldcg(p.part_ml + 2 * r + 1);
        if (l > 0.f) {
            const float ws = l * fast_exp2(m - M);
            num += ws * __ldcg(p.part_o + r * ATT_D + d);
            den += ws;
        }
    }
    const float o = den > 0.f ? num / den * p.v_scale[h] : 0.f;
    p.out[((int64_t)i * p.Hq + hq) * ATT_D + d] = __float2bfloat16_rn(o);
}

}  // namespace nvfp4sk
