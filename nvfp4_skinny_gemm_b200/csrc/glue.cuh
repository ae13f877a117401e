// glue.cuh -- small kernels of the verify step between the NVFP4 linears:
// FP8 KV-cache append of the tree nodes, and the per-row argmax of the
// LM-head logits.
#pragma once
#include "common.cuh"

namespace nvfp4sk {

// One CTA per (node i, KV head h); thread d writes K[d] and V[d] of that
// token as E4M3(fp32(x / scale[h])) into the paged pools.  K pages are
// token-major; a V (page, head) plane is cut into 8-dimension x 16-slot tiles
// of 128 bytes, tile (d/8, slot/16) at index (d/8)*(P/16) + slot/16, rows d%8
// of 16 slot bytes inside (the operand image the attention PV product reads).
__global__ void __launch_bounds__(128) kv_append_kernel(const __nv_bfloat16 *__restrict__ k_new,
                                                        const __nv_bfloat16 *__restrict__ v_new, int64_t ld_new,
                                                        int Hkv, int D, uint8_t *__restrict__ k_pool,
                                                        uint8_t *__restrict__ v_pool, int64_t n_pool_pages, int P,
                                                        const int32_t *__restrict__ page_table, int64_t ctx_len,
                                                        const float *__restrict__ k_scale,
                                                        const float *__restrict__ v_scale)
{
    pdl_wait();
    pdl_launch_dependents();
    const int i = blockIdx.x, h = blockIdx.y;
    const int64_t pos = ctx_len + i;
    const int32_t pg = page_table[pos / P];
    const int slot = (int)(pos % P);
    if (pg < 0 || pg >= n_pool_pages) {
        if (threadIdx.x == 0) report_error(ERRBIT_RANGE, 401);
        return;
    }
    const float ks = k_scale[h], vs = v_scale[h];
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        const float kx = __bfloat162float(k_new[(int64_t)i * ld_new + (int64_t)h * D + d]);
        const float vx = __bfloat162float(v_new[(int64_t)i * ld_new + (int64_t)h * D + d]);
        k_pool[(((int64_t)pg * Hkv + h) * P + slot) * D + d] = (uint8_t)(cvt_e4m3x2(__fdiv_rn(kx, ks), 0.f) & 0xFFu);
        const int64_t v_byte = ((int64_t)(d >> 3) * (P >> 4) + (slot >> 4)) * 128 + (d & 7) * 16 + (slot & 15);
        v_pool[((int64_t)pg * Hkv + h) * (int64_t)D * P + v_byte] = (uint8_t)(cvt_e4m3x2(__fdiv_rn(vx, vs), 0.f) & 0xFFu);
    }
}

// argmax over bf16 rows: grid (chunks, rows); each CTA reduces its chunk to
// (value, index), the last CTA of a row (arrival counter) reduces the chunk
// results in chunk order.  Ties resolve to the lowest index.
constexpr int AMX_THREADS = 256;

__device__ __forceinline__ bool amx_better(float v, int i, float bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(AMX_THREADS) argmax_rows_kernel(const __nv_bfloat16 *__restrict__ x, int64_t n,
                                                                   int64_t ld, int32_t *__restrict__ idx,
                                                                   float *__restrict__ part_v,
                                                                   int32_t *__restrict__ part_i,
                                                                   int32_t *__restrict__ counters)
{
    __shared__ float sv[AMX_THREADS / 32];
    __shared__ int si[AMX_THREADS / 32];
    __shared__ int s_last;
    pdl_wait();
    pdl_launch_dependents();
    const int r = blockIdx.y, ch = blockIdx.x, nch = gridDim.x;
    const int64_t per = (n + nch - 1) / nch;
    const int64_t j0 = (int64_t)ch * per, j1 = min(n, j0 + per);
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
    const __nv_bfloat16 *row = x + (int64_t)r * ld;
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        const float v = __bfloat162float(row[j]);
        if (amx_better(v, (int)j, bv, bi)) { bv = v; bi = (int)j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (amx_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane_id() == 0) { sv[warp_id()] = bv; si[warp_id()] = bi; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < AMX_THREADS / 32; ++w)
            if (amx_better(sv[w], si[w], bv, bi)) { bv = sv[w]; bi = si[w]; }
        part_v[(int64_t)r * nch + ch] = bv;
        part_i[(int64_t)r * nch + ch] = bi;
        __threadfence();
        s_last = atomicAdd(counters + r, 1) == nch - 1;
    }
    __syncthreads();
    if (s_last && threadIdx.x == 0) {
        __threadfence();
        float b = -INFINITY;
        int bidx = 0x7FFFFFFF;
        for (int k = 0; k < nch; ++k) {
            const float v = __ldcg(part_v + (int64_t)r * nch + k);
            const int i = __ldcg(part_i + (int64_t)r * nch + k);
            if (amx_better(v, i, b, bidx)) { b = v; bidx = i; }
        }
        idx[r] = bidx;
        counters[r] = 0;
    }
}

}  // namespace nvfp4sk
