// restore.cuh -- prefix-cache restore: dst page dst_ids[i] <- src page
// src_ids[i] as one gather-copy kernel.  Each CTA owns a strided set of
// chunks (<= 32 KB pieces of pages) and moves them with the bulk-copy engine:
// cp.async.bulk global->shared (mbarrier completion) and shared->global
// (bulk groups), a ring of stages deep enough to keep ~100 KB per SM in flight.
// One thread per CTA issues everything; the copy never touches registers.
#pragma once
#include "common.cuh"

namespace nvfp4sk {

constexpr int RST_THREADS = 32;
constexpr uint32_t RST_SMEM_BUDGET = 200 * 1024;
constexpr int RST_MAX_STAGES = 8;

struct RestoreParams {
    const uint8_t *src;
    const int32_t *src_ids;
    uint8_t *dst;
    const int32_t *dst_ids;
    int64_t n_items;          // n * chunks_per_page
    int64_t page_bytes;
    int64_t n_src_pages, n_dst_pages;
    uint32_t chunk;           // bytes per chunk (multiple of 16)
    int chunks_per_page;
    int stages;
};

__global__ void __launch_bounds__(RST_THREADS, 1) kv_page_restore_kernel(const RestoreParams p)
{
    extern __shared__ uint8_t rst_smem_raw[];
    uint8_t *buf = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rst_smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(buf + (size_t)p.stages * p.chunk);
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x != 0) return;
    for (int s = 0; s < p.stages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();

    // items of this CTA: it = blockIdx.x + k * gridDim.x
    const int64_t G = gridDim.x;
    const int64_t n_my = p.n_items > blockIdx.x ? (p.n_items - blockIdx.x + G - 1) / G : 0;
    auto item_src_dst = [&](int64_t k, const uint8_t *&s, uint8_t *&d, uint32_t &bytes) -> bool {
        const int64_t it = blockIdx.x + k * G;
        const int64_t i = it / p.chunks_per_page, ch = it % p.chunks_per_page;
        const int32_t si = p.src_ids[i], di = p.dst_ids[i];
        const int64_t off = ch * (int64_t)p.chunk;
        const int64_t rem = p.page_bytes - off;
        bytes = (uint32_t)(rem < (int64_t)p.chunk ? rem : (int64_t)p.chunk);
        if (si < 0 || si >= p.n_src_pages || di < 0 || di >= p.n_dst_pages) {
            report_error(ERRBIT_RANGE, 201);
            return false;
        }
        s = p.src + (int64_t)si * p.page_bytes + off;
        d = p.dst + (int64_t)di * p.page_bytes + off;
        return true;
    };
    auto issue_load = [&](int64_t k) {
        const int st = (int)(k % p.stages);
        const uint8_t *s; uint8_t *d; uint32_t bytes;
        if (item_src_dst(k, s, d, bytes)) {
            mbar_arrive_expect_tx(&full[st], bytes);
            bulk_load(buf + (size_t)st * p.chunk, s, bytes, &full[st]);
        } else {
            mbar_arrive(&full[st]);   // invalid ids: complete the phase, copy nothing
        }
    };
    const int64_t pre = n_my < p.stages - 1 ? n_my : p.stages - 1;
    for (int64_t k = 0; k < pre; ++k) issue_load(k);
    for (int64_t k = 0; k < n_my; ++k) {
        const int st = (int)(k % p.stages);
        if (!mbar_wait(&full[st], (uint32_t)((k / p.stages) & 1), 202)) {
            // give up: let the loads already issued (items k .. k+stages-2) land first
            for (int64_t j = k + 1; j < n_my && j < k + p.stages - 1; ++j)
                mbar_wait(&full[j % p.stages], (uint32_t)((j / p.stages) & 1), 203);
            break;
        }
        const uint8_t *s; uint8_t *d; uint32_t bytes;
        if (item_src_dst(k, s, d, bytes)) bulk_store(d, buf + (size_t)st * p.chunk, bytes);
        bulk_commit();
        // the next load reuses the stage of item k-1: its store must have read smem
        bulk_wait_read<1>();
        if (k + p.stages - 1 < n_my) issue_load(k + p.stages - 1);
    }
    bulk_wait<0>();
}

}  // namespace nvfp4sk
