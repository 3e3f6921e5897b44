// gqa_decode_noalloc: gqa_decode for callers that cannot provide a workspace.
//
// Some callers have no way to allocate device memory for the decode workspace: a plugin hosted
// by a framework that owns every device allocation and hands out only the tensors it manages,
// or a serving loop that must not call cudaMalloc (which can synchronize the whole device) and
// has no spare buffer of its own to lend.  For them this file keeps the workspace in a fixed
// array of device memory that belongs to the library itself, and forwards to gqa_decode.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds its
// kScratchBytes until the process exits.  In host code its name is only a host-side stand-in,
// so the device address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, and cached.
#include <cuda_runtime_api.h>

#include <mutex>

#include "gqa.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = GQA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on first use).
int scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return GQA_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices) return GQA_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return GQA_OK;
}

}  // namespace

extern "C" int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                                  int L_max, float scale, gqa_dtype_t dtype, float *out,
                                  int32_t *status, cudaStream_t stream) {
    const size_t need = gqa_decode_workspace_size(B, H_q, H_kv, d, dtype);
    if (need > kScratchBytes) return GQA_ERR_SCRATCH_LIMIT;
    // Every other host-side check of gqa_decode (pointers, alignment, sizes, element type,
    // scale, device), before anything is queued on the stream; need == 0 (invalid sizes or no
    // usable device) is reported here with gqa_decode's own code.
    int rc = gqa::decode_check(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, scale,
                               dtype, out, status);
    if (rc != GQA_OK) return rc;
    if (need == 0) return GQA_ERR_SHAPE;  // not reached: decode_check refuses those sizes
    void *ws = nullptr;
    rc = scratch_address(&ws);
    if (rc != GQA_OK) return rc;
    // The workspace's piece counters must be zero; a call that timed out may have left some
    // set, and the caller cannot reach this array, so clear them on the stream every time.
    size_t off = 0;
    const size_t cnt_bytes = gqa::decode_counter_region(B, H_q, H_kv, d, &off);
    if (cnt_bytes > 0 && cudaMemsetAsync(static_cast<unsigned char *>(ws) + off, 0, cnt_bytes, stream) != cudaSuccess)
        return GQA_ERR_CUDA;
    return gqa_decode(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, scale, dtype, out,
                      ws, kScratchBytes, status, stream);
}
