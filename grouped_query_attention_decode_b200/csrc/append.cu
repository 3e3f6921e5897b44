// KV append of one decode step: write k_new/v_new into row seq_lens[b] of every key/value
// head of sequence b, then advance seq_lens[b] ("GQA 阅读笔记", Algorithm 2, the lines that
// write K_cache[t, g, :] and V_cache[t, g, :]).  In the [B][L_max][H_kv][d] layout the H_kv
// rows of one position are one contiguous block, so each sequence is two straight 16-byte
// vector copies.  One CTA per sequence.
#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"

namespace gqa {

// Appends `rows` consecutive rows per sequence (rows = 1 for one decode step; several for the
// drafted tokens of a speculative step), which form one contiguous block of the cache.
__global__ void __launch_bounds__(128)
append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint4 *k_cache,
              uint4 *v_cache, int32_t *seq_lens, int H_kv, int row_vecs, int L_max, int rows,
              int32_t *status) {
    const int b = blockIdx.x;
    const int t = seq_lens[b];
    // Let a following decode launch start its prologue while this copy runs.
    grid_launch_dependents();
    __syncthreads();  // every thread has read seq_lens[b] before thread 0 advances it
    if (t < 0 || t > L_max - rows) {
        if (threadIdx.x == 0 && status != nullptr) atomicOr(status, GQA_STATUS_APPEND_OVERFLOW);
        return;
    }
    const long long row = static_cast<long long>(H_kv) * row_vecs;  // 16-byte vectors per row
    const long long blk = row * rows;
    const uint4 *ks = k_new + b * blk;
    const uint4 *vs = v_new + b * blk;
    uint4 *kd = k_cache + (static_cast<long long>(b) * L_max + t) * row;
    uint4 *vd = v_cache + (static_cast<long long>(b) * L_max + t) * row;
    for (long long i = threadIdx.x; i < blk; i += blockDim.x) {
        kd[i] = ks[i];
        vd[i] = vs[i];
    }
    if (threadIdx.x == 0) seq_lens[b] = t + rows;
}

// Paged variant: row t = seq_lens[b] goes to row t % page_size of page
// block_table[b * max_pages + t / page_size] of the pool [n_pages][page_size][H_kv][d].
__global__ void __launch_bounds__(128)
append_paged_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                    uint4 *k_pool, uint4 *v_pool, const int32_t *__restrict__ block_table,
                    int max_pages, int32_t *seq_lens, int H_kv, int row_vecs, int page_size,
                    int n_pages, int32_t *status) {
    const int b = blockIdx.x;
    const int t = seq_lens[b];
    grid_launch_dependents();
    __syncthreads();  // every thread has read seq_lens[b] before thread 0 advances it
    if (t < 0 || t >= max_pages * page_size) {
        if (threadIdx.x == 0 && status != nullptr) atomicOr(status, GQA_STATUS_APPEND_OVERFLOW);
        return;
    }
    const int page = block_table[static_cast<long long>(b) * max_pages + t / page_size];
    if (page < 0 || page >= n_pages) {
        if (threadIdx.x == 0 && status != nullptr) atomicOr(status, GQA_STATUS_APPEND_OVERFLOW);
        return;
    }
    const long long blk = static_cast<long long>(H_kv) * row_vecs;
    const uint4 *ks = k_new + b * blk;
    const uint4 *vs = v_new + b * blk;
    uint4 *kd = k_pool + (static_cast<long long>(page) * page_size + t % page_size) * blk;
    uint4 *vd = v_pool + (static_cast<long long>(page) * page_size + t % page_size) * blk;
    for (long long i = threadIdx.x; i < blk; i += blockDim.x) {
        kd[i] = ks[i];
        vd[i] = vs[i];
    }
    if (threadIdx.x == 0) seq_lens[b] = t + 1;
}

int launch_append_paged(const void *k_new, const void *v_new, void *k_pool, void *v_pool,
                        const int32_t *block_table, int max_pages, int32_t *seq_lens, int B,
                        int H_kv, int row_bytes, int page_size, int n_pages, int32_t *status,
                        cudaStream_t stream) {
    append_paged_kernel<<<B, 128, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
        static_cast<uint4 *>(k_pool), static_cast<uint4 *>(v_pool), block_table, max_pages,
        seq_lens, H_kv, row_bytes / 16, page_size, n_pages, status);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int launch_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  int32_t *seq_lens, int B, int H_kv, int row_bytes, int L_max, int rows,
                  int32_t *status, cudaStream_t stream) {
    append_kernel<<<B, 128, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), seq_lens, H_kv,
        row_bytes / 16, L_max, rows, status);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace gqa
