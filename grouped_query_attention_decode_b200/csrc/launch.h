// Host-side declarations shared by the kernel files and the C-ABI entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>

#include <cstdint>

#include "gqa.h"

namespace gqa {

struct DecodeParams;

// TMA descriptors of one bf16 decode call: q as [B*H_q rows][d], the caches as
// (d, H_kv, L_max, B) with 128-row and 8-row boxes of 64 columns, all with 128-byte swizzle.
struct TmaMaps {
    CUtensorMap q, k, k8, v, v8;
};

int launch_split_tc(const TmaMaps &maps, const DecodeParams &p, cudaStream_t stream);
int tc_q_box_rows(int heads_per_unit);
int tc_tile_rows(int d, int heads_per_unit);
int launch_split_f32(const DecodeParams &p, const float *q, const float *kc, const float *vc,
                     cudaStream_t stream);
// FP8 (e4m3) cache: the split kernel (K/V maps of uint8 codes with box rows tc8_tile_rows or
// the page size, and 8-row boxes; q is read from global memory) and the quantising append.
int tc8_tile_rows(int heads_per_unit);
// Byte offset and size of the per-unit piece counters inside a decode workspace for these
// sizes on the current device (0 bytes when the sizes are invalid).
size_t decode_counter_region(int B, int H_q, int H_kv, int d, size_t *offset);
// Every host-side check gqa_decode makes except those of the workspace, in the same order and
// with the same return codes; launches nothing.
int decode_check(const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                 int B, int H_q, int H_kv, int d, int L_max, float scale, gqa_dtype_t dtype,
                 float *out, int32_t *status);
int launch_split_tc8(const TmaMaps &maps, const void *q, const DecodeParams &p, cudaStream_t stream);
int launch_append_fp8(const void *k_new, const void *v_new, bool bf16_in, void *k_cache,
                      void *v_cache, const float *k_scale, const float *v_scale, int32_t *seq_lens,
                      const int32_t *block_table, int max_pages, int page_size, int n_pages,
                      int B, int H_kv, int d, int L_max, int rows, int32_t *status,
                      cudaStream_t stream);
int launch_append_paged(const void *k_new, const void *v_new, void *k_pool, void *v_pool,
                        const int32_t *block_table, int max_pages, int32_t *seq_lens, int B,
                        int H_kv, int row_bytes, int page_size, int n_pages, int32_t *status,
                        cudaStream_t stream);
int launch_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  int32_t *seq_lens, int B, int H_kv, int row_bytes, int L_max, int rows,
                  int32_t *status, cudaStream_t stream);

}  // namespace gqa
