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

// FP8 append: the new rows (bf16 or float32) become e4m3 codes of their head's scale,
// code = nearest e4m3 value of x / scale[g] (float32 division; ties to even; saturating at
// +-448), written at row seq_lens[b] of the contiguous cache or of the sequence's page.  The
// scaling reading is the FP8 cache of "GQA 阅读笔记", section "复现性与工程实践" (mixed
// precision): one float32 scale per key/value head for K and another for V.  One CTA per
// sequence; each thread quantises 16 consecutive elements (one head, one 16-byte store).
template <bool BF16_IN>
__global__ void __launch_bounds__(128)
append_fp8_kernel(const void *__restrict__ k_new, const void *__restrict__ v_new, uint8_t *k_cache,
                  uint8_t *v_cache, const float *__restrict__ k_scale,
                  const float *__restrict__ v_scale, int32_t *seq_lens,
                  const int32_t *__restrict__ block_table, int max_pages, int page_size,
                  int n_pages, int H_kv, int d, int L_max, int rows, int32_t *status) {
    const int b = blockIdx.x;
    const int t = seq_lens[b];
    grid_launch_dependents();
    __syncthreads();  // every thread has read seq_lens[b] before thread 0 advances it
    const bool paged = block_table != nullptr;
    const long long cap = paged ? static_cast<long long>(max_pages) * page_size : L_max;
    if (t < 0 || t > cap - rows) {
        if (threadIdx.x == 0 && status != nullptr) atomicOr(status, GQA_STATUS_APPEND_OVERFLOW);
        return;
    }
    const long long row_elems = static_cast<long long>(H_kv) * d;
    long long dst0;
    if (paged) {  // rows == 1
        const int page = block_table[static_cast<long long>(b) * max_pages + t / page_size];
        if (page < 0 || page >= n_pages) {
            if (threadIdx.x == 0 && status != nullptr) atomicOr(status, GQA_STATUS_APPEND_OVERFLOW);
            return;
        }
        dst0 = (static_cast<long long>(page) * page_size + t % page_size) * row_elems;
    } else {
        dst0 = (static_cast<long long>(b) * L_max + t) * row_elems;
    }
    const long long src0 = static_cast<long long>(b) * rows * row_elems;
    const long long chunks = rows * row_elems / 16;
    for (long long c = threadIdx.x; c < chunks; c += blockDim.x) {
        const long long e = c * 16;
        const int g = static_cast<int>((e / d) % H_kv);
        const float sk = k_scale[g], sv = v_scale[g];
        float kx[16], vx[16];
        if constexpr (BF16_IN) {
            const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(k_new) + src0 + e);
            const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(v_new) + src0 + e);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint4 a = ks[u], bv = vs[u];
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    kx[u * 8 + 2 * k] = __uint_as_float(aw[k] << 16);
                    kx[u * 8 + 2 * k + 1] = __uint_as_float(aw[k] & 0xFFFF0000u);
                    vx[u * 8 + 2 * k] = __uint_as_float(bw[k] << 16);
                    vx[u * 8 + 2 * k + 1] = __uint_as_float(bw[k] & 0xFFFF0000u);
                }
            }
        } else {
            const float4 *ks = reinterpret_cast<const float4 *>(static_cast<const float *>(k_new) + src0 + e);
            const float4 *vs = reinterpret_cast<const float4 *>(static_cast<const float *>(v_new) + src0 + e);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 a = ks[u], bv = vs[u];
                kx[4 * u] = a.x; kx[4 * u + 1] = a.y; kx[4 * u + 2] = a.z; kx[4 * u + 3] = a.w;
                vx[4 * u] = bv.x; vx[4 * u + 1] = bv.y; vx[4 * u + 2] = bv.z; vx[4 * u + 3] = bv.w;
            }
        }
        uint32_t kw[4], vw[4];
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
            const uint16_t k01 = e4m3x2_from_f32(__fdiv_rn(kx[k], sk), __fdiv_rn(kx[k + 1], sk));
            const uint16_t k23 = e4m3x2_from_f32(__fdiv_rn(kx[k + 2], sk), __fdiv_rn(kx[k + 3], sk));
            const uint16_t v01 = e4m3x2_from_f32(__fdiv_rn(vx[k], sv), __fdiv_rn(vx[k + 1], sv));
            const uint16_t v23 = e4m3x2_from_f32(__fdiv_rn(vx[k + 2], sv), __fdiv_rn(vx[k + 3], sv));
            kw[k / 4] = static_cast<uint32_t>(k01) | (static_cast<uint32_t>(k23) << 16);
            vw[k / 4] = static_cast<uint32_t>(v01) | (static_cast<uint32_t>(v23) << 16);
        }
        *reinterpret_cast<uint4 *>(k_cache + dst0 + e) = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        *reinterpret_cast<uint4 *>(v_cache + dst0 + e) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
    }
    if (threadIdx.x == 0) seq_lens[b] = t + rows;
}

int launch_append_fp8(const void *k_new, const void *v_new, bool bf16_in, void *k_cache,
                      void *v_cache, const float *k_scale, const float *v_scale, int32_t *seq_lens,
                      const int32_t *block_table, int max_pages, int page_size, int n_pages,
                      int B, int H_kv, int d, int L_max, int rows, int32_t *status,
                      cudaStream_t stream) {
    if (bf16_in)
        append_fp8_kernel<true><<<B, 128, 0, stream>>>(
            k_new, v_new, static_cast<uint8_t *>(k_cache), static_cast<uint8_t *>(v_cache), k_scale,
            v_scale, seq_lens, block_table, max_pages, page_size, n_pages, H_kv, d, L_max, rows, status);
    else
        append_fp8_kernel<false><<<B, 128, 0, stream>>>(
            k_new, v_new, static_cast<uint8_t *>(k_cache), static_cast<uint8_t *>(v_cache), k_scale,
            v_scale, seq_lens, block_table, max_pages, page_size, n_pages, H_kv, d, L_max, rows, status);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
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
