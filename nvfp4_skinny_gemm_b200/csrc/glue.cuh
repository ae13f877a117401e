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

// Token-major V planes -> the tiled plane layout the attention reads.  One CTA
// per (page, head) plane of P slots x D dimensions: the plane is staged in
// shared memory with 16-byte loads, then each 16-byte output row (dimension
// d, slots 16j .. 16j+15) is gathered from it and stored with one 16-byte
// write.  D % 8 == 0, P % 16 == 0, D * P <= KVT_MAX_PLANE.
constexpr int KVT_MAX_PLANE = 16384;
__global__ void __launch_bounds__(256) kv_v_to_tiled_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                                            int D, int P)
{
    __shared__ __align__(16) uint8_t plane[KVT_MAX_PLANE];
    pdl_wait();
    pdl_launch_dependents();
    const int64_t bytes = (int64_t)D * P;
    const uint8_t *s = src + blockIdx.x * bytes;
    uint8_t *o = dst + blockIdx.x * bytes;
    for (int64_t i = threadIdx.x; i < bytes / 16; i += blockDim.x)
        *reinterpret_cast<uint4 *>(plane + 16 * i) = *reinterpret_cast<const uint4 *>(s + 16 * i);
    __syncthreads();
    const int tiles_t = P / 16;
    for (int64_t row = threadIdx.x; row < bytes / 16; row += blockDim.x) {
        // output row `row`: tile (d / 8, j) = row / 8 with j fastest, line d % 8 = row % 8
        const int tile = (int)(row >> 3), d = (tile / tiles_t) * 8 + (int)(row & 7), j = tile % tiles_t;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t v = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) v |= (uint32_t)plane[(16 * j + 4 * q + b) * D + d] << (8 * b);
            w[q] = v;
        }
        *reinterpret_cast<uint4 *>(o + 16 * row) = make_uint4(w[0], w[1], w[2], w[3]);
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

namespace nvfp4sk {

// ---- greedy acceptance of the verified tree -------------------------------
// One warp.  Node 0 (the root: the last accepted token) is accepted; node
// i >= 1 is accepted when its parent is accepted and its draft token equals
// the target's greedy choice after the parent.  The accepted path runs from
// the root to the deepest accepted node (lowest index among equally deep
// ones); the next token is the target's choice after that node.  A parent
// array that is not topologically ordered (parent[0] != -1, or parent[i]
// outside [0, i)) is flagged (site 501) and only the root is accepted.
constexpr int ACC_MAX_T = 32;

__global__ void __launch_bounds__(32) tree_accept_kernel(const int32_t *__restrict__ tok,
                                                         const int32_t *__restrict__ amax,
                                                         const int32_t *__restrict__ parent, int T,
                                                         int32_t *__restrict__ path, int32_t *__restrict__ n_acc,
                                                         int32_t *__restrict__ next_tok)
{
    __shared__ int s_par[ACC_MAX_T], s_tok[ACC_MAX_T], s_amax[ACC_MAX_T];
    pdl_wait();
    pdl_launch_dependents();
    const int i = threadIdx.x;
    if (i < T) {
        s_par[i] = parent[i];
        s_tok[i] = tok[i];
        s_amax[i] = amax[i];
    }
    __syncwarp();
    if (i != 0) return;
    bool bad = s_par[0] != -1;
    for (int j = 1; j < T; ++j) bad |= s_par[j] < 0 || s_par[j] >= j;
    uint32_t acc_mask = 1u;
    int depth[ACC_MAX_T];
    depth[0] = 0;
    int end = 0;
    if (!bad) {
        for (int j = 1; j < T; ++j) {
            const int p = s_par[j];
            depth[j] = depth[p] + 1;
            if (((acc_mask >> p) & 1u) && s_tok[j] == s_amax[p]) {
                acc_mask |= 1u << j;
                if (depth[j] > depth[end]) end = j;
            }
        }
    } else {
        report_error(ERRBIT_RANGE, 501);
    }
    const int n = depth[end] + 1;
    for (int k = n - 1, a = end; k >= 0; --k, a = k >= 0 ? s_par[a] : a) path[k] = a;
    *n_acc = n;
    *next_tok = s_amax[end];
}

// ---- move the accepted tokens' K/V next to the context --------------------
// Grid (layers, KV heads), one thread per dimension: the K and V bytes of the
// accepted path's tokens (tree slots ctx_len + path[k]) are read first, then
// written to positions ctx_len + k, in every layer.
__global__ void __launch_bounds__(128) kv_compact_kernel(uint8_t *__restrict__ k_base, uint8_t *__restrict__ v_base,
                                                         int64_t layer_stride, int Hkv, int D,
                                                         int64_t n_pool_pages, int P,
                                                         const int32_t *__restrict__ page_table, int64_t ctx_len,
                                                         const int32_t *__restrict__ path,
                                                         const int32_t *__restrict__ n_acc, int T)
{
    pdl_wait();
    pdl_launch_dependents();
    const int l = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
    const int n = min(max(*n_acc, 0), T);
    uint8_t *kp = k_base + (int64_t)l * layer_stride, *vp = v_base + (int64_t)l * layer_stride;
    uint8_t kr[ACC_MAX_T], vr[ACC_MAX_T];
    bool ok = true;
    auto locate = [&](int64_t pos, int64_t &pg, int &slot) {
        pg = page_table[pos / P];
        slot = (int)(pos % P);
        return pg >= 0 && pg < n_pool_pages;
    };
#pragma unroll 1
    for (int k = 0; k < n; ++k) {
        const int node = path[k];
        int64_t pg;
        int slot;
        if (node < 0 || node >= T || !locate(ctx_len + node, pg, slot)) {
            if (d == 0) report_error(ERRBIT_RANGE, 502);
            ok = false;
            break;
        }
        if (d < D) {
            kr[k] = kp[((pg * Hkv + h) * P + slot) * D + d];
            vr[k] = vp[(pg * Hkv + h) * (int64_t)D * P + ((d >> 3) * (P >> 4) + (slot >> 4)) * 128 + (d & 7) * 16 + (slot & 15)];
        }
    }
    __syncthreads();
    if (!__syncthreads_and(ok ? 1 : 0)) return;
#pragma unroll 1
    for (int k = 0; k < n; ++k) {
        int64_t pg;
        int slot;
        if (!locate(ctx_len + k, pg, slot)) {
            if (d == 0) report_error(ERRBIT_RANGE, 502);
            return;
        }
        if (d < D) {
            kp[((pg * Hkv + h) * P + slot) * D + d] = kr[k];
            vp[(pg * Hkv + h) * (int64_t)D * P + ((d >> 3) * (P >> 4) + (slot >> 4)) * 128 + (d & 7) * 16 + (slot & 15)] = vr[k];
        }
    }
}

}  // namespace nvfp4sk
