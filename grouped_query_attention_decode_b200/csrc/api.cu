// C-ABI entry points of libgqa (declared and documented in include/gqa.h): argument checks,
// workspace sizing, TMA descriptor encoding and kernel launches.  No device memory is
// allocated here.
#include <cuda.h>
#include <cuda_runtime_api.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {
namespace {

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};
std::atomic<cudaEvent_t> g_ev_before{nullptr};
std::atomic<cudaEvent_t> g_ev_after{nullptr};

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// SM count of the current device, or <= 0 when there is none (or it is not sm_100).
int current_sm_count(int *dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 0;
    }
    *dev_out = dev;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sm_count[dev] == 0) {
        int sms = 0, major = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        g_sm_count[dev] = (major == 10) ? sms : -1;
    }
    return g_sm_count[dev];
}

struct Geometry {
    int r, rb, RB, HB, UB;
    long long units, slots, slot_floats, slot_base;
    size_t bytes;
};

// Units: (sequence, key/value head, block of rb query heads) with Q query tokens each; a unit
// has RB = Q * rb <= kMaxUnitCols columns.  A group of more than 32 query heads is cut into
// blocks of 32 that read the same K/V tiles (the second read of a tile finds it in L2 when the
// blocks' pieces run close together), which keeps every softmax thread's per-column state in
// registers.
constexpr int kMaxUnitCols = 32;
Geometry geometry(int B, int H_q, int H_kv, int d, int G, int Q = 1) {
    Geometry g;
    g.r = H_q / H_kv;
    g.rb = g.r < kMaxUnitCols / Q ? g.r : kMaxUnitCols / Q;
    g.RB = Q * g.rb;
    g.HB = (g.r + g.rb - 1) / g.rb;
    g.UB = H_kv * g.HB;
    g.units = static_cast<long long>(B) * g.UB;
    g.slots = G + g.units - 1;
    // O [RB][d], m [RB], l [RB], rounded up to whole 16-byte vectors (the merge reads o with
    // 16-byte loads)
    g.slot_floats = (static_cast<long long>(g.RB) * (d + 2) + 3) / 4 * 4;
    // the per-unit piece counters (int32, kPieceGroups per unit) at offset 0, then the slots
    // from the next 256-byte boundary
    g.slot_base = (g.units * kPieceGroups * 4 + 255) / 256 * 64;
    g.bytes = static_cast<size_t>((g.slot_base + g.slots * g.slot_floats) * 4 + 255) / 256 * 256;
    return g;
}

int check_shape(int B, int H_q, int H_kv, int d, int L_max, gqa_dtype_t dtype,
                bool allow_e4m3 = false) {
    if (dtype != GQA_DTYPE_F32 && dtype != GQA_DTYPE_BF16 &&
        !(allow_e4m3 && dtype == GQA_DTYPE_E4M3))
        return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || H_q <= 0 || H_kv <= 0 || L_max <= 0) return GQA_ERR_SHAPE;
    if (H_q % H_kv != 0) return GQA_ERR_HEADS_NOT_DIVISIBLE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    // Index arithmetic in the kernels: rows of q and tiles per launch stay well inside int32.
    if (static_cast<long long>(B) * H_q > (1ll << 30) || static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    return GQA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

bool encode_cache_map(CUtensorMap *m, const void *base, int B, int H_kv, int d, int L_max, int rows) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv),
                                static_cast<cuuint64_t>(L_max), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(H_kv) * d * 2,
                                   static_cast<cuuint64_t>(L_max) * H_kv * d * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B,
                       // L2 fetches as wide as a cached row of one head: 256 bytes would also bring
                       // the next head's half of a 128-byte row, which another CTA reads later
                       d == 64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An e4m3 cache as (d, H_kv, rows, sequences or pages) of bytes; boxes of `rows` rows of one
// key/value head, d bytes wide, swizzled as the UMMA operands expect (128-byte swizzle for
// d = 128, 64-byte for d = 64).
bool encode_cache_map8(CUtensorMap *m, const void *base, int outer, int H_kv, int d, int rows_dim,
                       int rows) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv),
                                static_cast<cuuint64_t>(rows_dim), static_cast<cuuint64_t>(outer)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d),
                                   static_cast<cuuint64_t>(H_kv) * d,
                                   static_cast<cuuint64_t>(rows_dim) * H_kv * d};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(d), 1, static_cast<cuuint32_t>(rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B,  // a row is at most 128 bytes
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q as (d, H_q, B*Q); one unit's tile is the box (64 columns, rb heads, Q tokens), which lands
// in shared memory as rows j * rb + h'.
bool encode_q_map(CUtensorMap *m, const void *q, int B, int Q, int H_q, int d, int rb) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_q),
                                static_cast<cuuint64_t>(B) * Q};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                   static_cast<cuuint64_t>(H_q) * d * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rb), static_cast<cuuint32_t>(Q)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace gqa

using namespace gqa;

extern "C" int gqa_kv_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                             int32_t *seq_lens, int B, int H_kv, int d, int L_max,
                             gqa_dtype_t dtype, int32_t *status, cudaStream_t stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !seq_lens) return GQA_ERR_NULL;
    if (dtype != GQA_DTYPE_F32 && dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || H_kv <= 0 || L_max <= 0 || static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(seq_lens, 4) || (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return GQA_ERR_NO_DEVICE;
    const int row_bytes = d * (dtype == GQA_DTYPE_BF16 ? 2 : 4);
    return launch_append(k_new, v_new, k_cache, v_cache, seq_lens, B, H_kv, row_bytes, L_max, 1,
                         status, stream);
}

extern "C" int gqa_kv_append_multi(const void *k_new, const void *v_new, void *k_cache,
                                   void *v_cache, int32_t *seq_lens, int B, int Q, int H_kv,
                                   int d, int L_max, gqa_dtype_t dtype, int32_t *status,
                                   cudaStream_t stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !seq_lens) return GQA_ERR_NULL;
    if (dtype != GQA_DTYPE_F32 && dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || Q <= 0 || Q > kMaxUnitCols || H_kv <= 0 || L_max <= 0 ||
        static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(seq_lens, 4) || (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return GQA_ERR_NO_DEVICE;
    const int row_bytes = d * (dtype == GQA_DTYPE_BF16 ? 2 : 4);
    return launch_append(k_new, v_new, k_cache, v_cache, seq_lens, B, H_kv, row_bytes, L_max, Q,
                         status, stream);
}

extern "C" size_t gqa_decode_multi_workspace_size(int B, int Q, int H_q, int H_kv, int d,
                                                  gqa_dtype_t dtype) {
    if (Q < 1 || Q > kMaxUnitCols || check_shape(B, H_q, H_kv, d, 1, dtype) != GQA_OK) return 0;
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return 0;
    return geometry(B, H_q, H_kv, d, sms, Q).bytes;
}

size_t gqa::decode_counter_region(int B, int H_q, int H_kv, int d, size_t *offset) {
    if (check_shape(B, H_q, H_kv, d, 1, GQA_DTYPE_BF16) != GQA_OK) return 0;
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return 0;
    const Geometry g = geometry(B, H_q, H_kv, d, sms);
    *offset = 0;
    return static_cast<size_t>(g.slot_base) * 4;
}

extern "C" size_t gqa_decode_workspace_size(int B, int H_q, int H_kv, int d, gqa_dtype_t dtype) {
    if (check_shape(B, H_q, H_kv, d, 1, dtype, true) != GQA_OK) return 0;
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return 0;
    return geometry(B, H_q, H_kv, d, sms).bytes;
}

namespace {

// Paged cache description for decode_impl (block_table == nullptr: contiguous caches).
struct PagedArgs {
    const int32_t *block_table = nullptr;
    int max_pages = 0, page_size = 0, n_pages = 0;
};

// The append fused into the decode (k_new == nullptr: none).
struct AppendArgs {
    const void *k_new = nullptr, *v_new = nullptr;
    void *k_cache = nullptr, *v_cache = nullptr;
    int32_t *lens_out = nullptr;
};

int decode_impl(const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
                int B, int H_q, int H_kv, int d, int L_max, int window, float scale,
                gqa_dtype_t dtype, float *out, void *workspace, size_t workspace_bytes,
                int32_t *status, cudaStream_t stream, const PagedArgs &pg = PagedArgs(),
                int Q = 1, const float *k_scale = nullptr, const float *v_scale = nullptr,
                bool dry_run = false, const AppendArgs &ap = AppendArgs()) {
    if (!q || !k_cache || !v_cache || !seq_lens || !out) return GQA_ERR_NULL;
    const bool fp8 = k_scale != nullptr;
    const int rc = check_shape(B, H_q, H_kv, d, L_max, dtype, fp8);
    if (rc != GQA_OK) return rc;
    if (fp8 && (dtype != GQA_DTYPE_E4M3 || !v_scale)) return GQA_ERR_NULL;
    if (fp8 && (!aligned(k_scale, 4) || !aligned(v_scale, 4))) return GQA_ERR_ALIGNMENT;
    if (!workspace) return GQA_ERR_WORKSPACE;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(seq_lens, 4) || !aligned(workspace, 256) || (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    if (!std::isfinite(scale)) return GQA_ERR_SHAPE;
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (sms <= 0) return GQA_ERR_NO_DEVICE;
    if (Q < 1 || Q > kMaxUnitCols) return GQA_ERR_SHAPE;
    const Geometry g = geometry(B, H_q, H_kv, d, sms, Q);
    if (workspace_bytes < g.bytes) return GQA_ERR_WORKSPACE;
    if (g.slot_floats % 4 != 0 || g.slot_base % 4 != 0) return GQA_ERR_SHAPE;  // 16-byte slot vectors

    DecodeParams p;
    p.seq_lens = seq_lens;
    p.out = out;
    p.ws = static_cast<float *>(workspace);
    p.status = status;
    p.B = B;
    p.H_q = H_q;
    p.H_kv = H_kv;
    p.d = d;
    p.L_max = L_max;
    p.r = g.r;
    p.Q = Q;
    p.rb = g.rb;
    p.q_box_bytes = (d / 64) * Q * g.rb * 128;
    p.RB = g.RB;
    p.HB = g.HB;
    p.UB = g.UB;
    p.T = fp8 ? tc8_tile_rows(g.RB) : (dtype == GQA_DTYPE_BF16 ? tc_tile_rows(d, g.RB) : 64);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_new = ap.k_new;
    p.v_new = ap.v_new;
    p.k_cache = ap.k_cache;
    p.v_cache = ap.v_cache;
    p.lens_out = ap.lens_out;
    p.append = ap.k_new != nullptr ? 1 : 0;
    p.window = window;
    p.block_table = pg.block_table;
    p.max_pages = pg.max_pages;
    p.page_size = pg.page_size;
    p.n_pages = pg.n_pages;
    // One persistent CTA per SM, but never more CTAs than the largest possible tile count
    // (the workspace is sized for one per SM, which bounds this).
    const long long span = (window > 0 && window < L_max) ? window : L_max;
    const long long max_tiles = g.units * ((span + p.T - 1) / p.T);
    p.G = max_tiles < sms ? static_cast<int>(max_tiles) : sms;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.wait_ns = g_wait_ns.load();
    p.slot_floats = g.slot_floats;
    p.slot_base = g.slot_base;
    p.cnt = static_cast<int32_t *>(workspace);

    cudaEvent_t ev0 = g_ev_before.load(), ev1 = g_ev_after.load();
    const bool profile = ev0 != nullptr && ev1 != nullptr;
    int res;
    if (fp8) {
        if (encode_fn() == nullptr) return GQA_ERR_CUDA;
        TmaMaps maps;
        const int rows_dim = pg.block_table ? pg.page_size : L_max;
        const int outer_dim = pg.block_table ? pg.n_pages : B;
        const int box = pg.block_table ? (pg.page_size < p.T ? pg.page_size : p.T) : p.T;
        if (!encode_cache_map8(&maps.k, k_cache, outer_dim, H_kv, d, rows_dim, box) ||
            !encode_cache_map8(&maps.k8, k_cache, outer_dim, H_kv, d, rows_dim, 8) ||
            !encode_cache_map8(&maps.v, v_cache, outer_dim, H_kv, d, rows_dim, box) ||
            !encode_cache_map8(&maps.v8, v_cache, outer_dim, H_kv, d, rows_dim, 8))
            return GQA_ERR_SHAPE;
        if (dry_run) return GQA_OK;
        if (profile && cudaEventRecord(ev0, stream) != cudaSuccess) return GQA_ERR_CUDA;
        res = launch_split_tc8(maps, q, p, stream);
    } else if (dtype == GQA_DTYPE_BF16) {
        const int rp = tc_q_box_rows(g.RB);
        if (encode_fn() == nullptr) return GQA_ERR_CUDA;
        TmaMaps maps;
        // The cache as (d, H_kv, rows, sequences) -- or, paged, (d, H_kv, page_size, n_pages).
        const int rows_dim = pg.block_table ? pg.page_size : L_max;
        const int outer_dim = pg.block_table ? pg.n_pages : B;
        const int box = pg.block_table ? (pg.page_size < p.T ? pg.page_size : p.T) : p.T;
        (void)rp;
        if (!encode_q_map(&maps.q, q, B, Q, H_q, d, g.rb) ||
            !encode_cache_map(&maps.k, k_cache, outer_dim, H_kv, d, rows_dim, box) ||
            !encode_cache_map(&maps.k8, k_cache, outer_dim, H_kv, d, rows_dim, 8) ||
            !encode_cache_map(&maps.v, v_cache, outer_dim, H_kv, d, rows_dim, box) ||
            !encode_cache_map(&maps.v8, v_cache, outer_dim, H_kv, d, rows_dim, 8))
            return GQA_ERR_SHAPE;
        if (dry_run) return GQA_OK;
        if (profile && cudaEventRecord(ev0, stream) != cudaSuccess) return GQA_ERR_CUDA;
        res = launch_split_tc(maps, p, stream);
    } else {
        if (dry_run) return GQA_OK;
        if (profile && cudaEventRecord(ev0, stream) != cudaSuccess) return GQA_ERR_CUDA;
        res = launch_split_f32(p, static_cast<const float *>(q), static_cast<const float *>(k_cache),
                               static_cast<const float *>(v_cache), stream);
    }
    if (res != GQA_OK) return res;
    if (profile && cudaEventRecord(ev1, stream) != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}

}  // namespace

int gqa::decode_check(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                      float scale, gqa_dtype_t dtype, float *out, int32_t *status) {
    // A stand-in workspace, never dereferenced: every check but the workspace's runs, and
    // nothing is launched.
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, 0, scale, dtype,
                       out, reinterpret_cast<void *>(static_cast<uintptr_t>(256)), SIZE_MAX, status,
                       nullptr, PagedArgs(), 1, nullptr, nullptr, true);
}

extern "C" int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                          float scale, gqa_dtype_t dtype, float *out, void *workspace,
                          size_t workspace_bytes, int32_t *status, cudaStream_t stream) {
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, 0, scale, dtype,
                       out, workspace, workspace_bytes, status, stream);
}

extern "C" int gqa_kv_append_decode(const void *q, const void *k_new, const void *v_new,
                                    void *k_cache, void *v_cache, const int32_t *seq_lens,
                                    int32_t *seq_lens_out, int B, int H_q, int H_kv, int d,
                                    int L_max, float scale, gqa_dtype_t dtype, float *out,
                                    void *workspace, size_t workspace_bytes, int32_t *status,
                                    cudaStream_t stream) {
    if (!k_new || !v_new || !seq_lens_out) return GQA_ERR_NULL;
    if (dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(seq_lens_out, 4))
        return GQA_ERR_ALIGNMENT;
    if (B > 0 && seq_lens != nullptr) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(seq_lens), b0 = reinterpret_cast<uintptr_t>(seq_lens_out);
        const uintptr_t n = static_cast<uintptr_t>(B) * sizeof(int32_t);
        if (a0 < b0 + n && b0 < a0 + n) return GQA_ERR_OVERLAP;
    }
    AppendArgs ap;
    ap.k_new = k_new;
    ap.v_new = v_new;
    ap.k_cache = k_cache;
    ap.v_cache = v_cache;
    ap.lens_out = seq_lens_out;
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, 0, scale, dtype, out,
                       workspace, workspace_bytes, status, stream, PagedArgs(), 1, nullptr, nullptr,
                       false, ap);
}

extern "C" int gqa_kv_append_paged(const void *k_new, const void *v_new, void *k_pool,
                                   void *v_pool, const int32_t *block_table, int max_pages,
                                   int32_t *seq_lens, int B, int H_kv, int d, int page_size,
                                   int n_pages, gqa_dtype_t dtype, int32_t *status,
                                   cudaStream_t stream) {
    if (!k_new || !v_new || !k_pool || !v_pool || !block_table || !seq_lens) return GQA_ERR_NULL;
    if (dtype != GQA_DTYPE_F32 && dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || H_kv <= 0 || max_pages <= 0 || n_pages <= 0 || page_size <= 0 ||
        page_size % 8 != 0 || static_cast<long long>(max_pages) * page_size > (1ll << 30) ||
        static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) ||
        !aligned(v_pool, 16) || !aligned(seq_lens, 4) || !aligned(block_table, 4) ||
        (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return GQA_ERR_NO_DEVICE;
    const int row_bytes = d * (dtype == GQA_DTYPE_BF16 ? 2 : 4);
    return launch_append_paged(k_new, v_new, k_pool, v_pool, block_table, max_pages, seq_lens, B,
                               H_kv, row_bytes, page_size, n_pages, status, stream);
}

extern "C" int gqa_decode_paged(const void *q, const void *k_pool, const void *v_pool,
                                const int32_t *block_table, int max_pages,
                                const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                                int page_size, int n_pages, float scale, gqa_dtype_t dtype,
                                float *out, void *workspace, size_t workspace_bytes,
                                int32_t *status, cudaStream_t stream) {
    if (!block_table) return GQA_ERR_NULL;
    if (!aligned(block_table, 4)) return GQA_ERR_ALIGNMENT;
    if (max_pages <= 0 || n_pages <= 0 || page_size <= 0 || page_size % 8 != 0 ||
        static_cast<long long>(max_pages) * page_size > (1ll << 30))
        return GQA_ERR_SHAPE;
    // a tile (128 rows, or 256 for 64-wide heads of groups up to 8) must lie in one page or
    // cover whole pages
    if (dtype == GQA_DTYPE_BF16 && H_kv > 0 && H_q % H_kv == 0) {
        const int tr = tc_tile_rows(d, H_q / H_kv < 32 ? H_q / H_kv : 32);
        if (tr % page_size != 0 && page_size % tr != 0) return GQA_ERR_SHAPE;
    }
    PagedArgs pg;
    pg.block_table = block_table;
    pg.max_pages = max_pages;
    pg.page_size = page_size;
    pg.n_pages = n_pages;
    return decode_impl(q, k_pool, v_pool, seq_lens, B, H_q, H_kv, d, max_pages * page_size, 0,
                       scale, dtype, out, workspace, workspace_bytes, status, stream, pg);
}

extern "C" int gqa_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *seq_lens, int B, int Q, int H_q, int H_kv, int d,
                                int L_max, float scale, gqa_dtype_t dtype, float *out,
                                void *workspace, size_t workspace_bytes, int32_t *status,
                                cudaStream_t stream) {
    if (Q < 1 || Q > kMaxUnitCols) return GQA_ERR_SHAPE;
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, 0, scale, dtype,
                       out, workspace, workspace_bytes, status, stream, PagedArgs(), Q);
}

extern "C" int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache,
                                 const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                                 int L_max, int window, float scale, gqa_dtype_t dtype,
                                 float *out, void *workspace, size_t workspace_bytes,
                                 int32_t *status, cudaStream_t stream) {
    if (window <= 0) return GQA_ERR_SHAPE;
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, window, scale,
                       dtype, out, workspace, workspace_bytes, status, stream);
}

extern "C" int gqa_kv_append_fp8(const void *k_new, const void *v_new, gqa_dtype_t new_dtype,
                                 void *k_cache, void *v_cache, const float *k_scale,
                                 const float *v_scale, int32_t *seq_lens, int B, int H_kv, int d,
                                 int L_max, int32_t *status, cudaStream_t stream) {
    if (!k_new || !v_new || !k_cache || !v_cache || !k_scale || !v_scale || !seq_lens)
        return GQA_ERR_NULL;
    if (new_dtype != GQA_DTYPE_F32 && new_dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || H_kv <= 0 || L_max <= 0 || static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(k_scale, 4) || !aligned(v_scale, 4) ||
        !aligned(seq_lens, 4) || (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return GQA_ERR_NO_DEVICE;
    return launch_append_fp8(k_new, v_new, new_dtype == GQA_DTYPE_BF16, k_cache, v_cache, k_scale,
                             v_scale, seq_lens, nullptr, 0, 0, 0, B, H_kv, d, L_max, 1, status,
                             stream);
}

extern "C" int gqa_kv_append_paged_fp8(const void *k_new, const void *v_new, gqa_dtype_t new_dtype,
                                       void *k_pool, void *v_pool, const float *k_scale,
                                       const float *v_scale, const int32_t *block_table,
                                       int max_pages, int32_t *seq_lens, int B, int H_kv, int d,
                                       int page_size, int n_pages, int32_t *status,
                                       cudaStream_t stream) {
    if (!k_new || !v_new || !k_pool || !v_pool || !k_scale || !v_scale || !block_table || !seq_lens)
        return GQA_ERR_NULL;
    if (new_dtype != GQA_DTYPE_F32 && new_dtype != GQA_DTYPE_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
    if (B <= 0 || H_kv <= 0 || max_pages <= 0 || n_pages <= 0 || page_size <= 0 ||
        page_size % 8 != 0 || static_cast<long long>(max_pages) * page_size > (1ll << 30) ||
        static_cast<long long>(B) * H_kv > (1ll << 30))
        return GQA_ERR_SHAPE;
    if (d != 64 && d != 128) return GQA_ERR_UNSUPPORTED_DIM;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) ||
        !aligned(v_pool, 16) || !aligned(k_scale, 4) || !aligned(v_scale, 4) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4) || (status && !aligned(status, 4)))
        return GQA_ERR_ALIGNMENT;
    int dev = 0;
    if (current_sm_count(&dev) <= 0) return GQA_ERR_NO_DEVICE;
    return launch_append_fp8(k_new, v_new, new_dtype == GQA_DTYPE_BF16, k_pool, v_pool, k_scale,
                             v_scale, seq_lens, block_table, max_pages, page_size, n_pages, B,
                             H_kv, d, 0, 1, status, stream);
}

extern "C" int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache,
                              const float *k_scale, const float *v_scale, const int32_t *seq_lens,
                              int B, int H_q, int H_kv, int d, int L_max, int window, float scale,
                              float *out, void *workspace, size_t workspace_bytes,
                              int32_t *status, cudaStream_t stream) {
    if (!k_scale || !v_scale) return GQA_ERR_NULL;
    if (window < 0) return GQA_ERR_SHAPE;
    return decode_impl(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, window, scale,
                       GQA_DTYPE_E4M3, out, workspace, workspace_bytes, status, stream,
                       PagedArgs(), 1, k_scale, v_scale);
}

extern "C" int gqa_decode_paged_fp8(const void *q, const void *k_pool, const void *v_pool,
                                    const float *k_scale, const float *v_scale,
                                    const int32_t *block_table, int max_pages,
                                    const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                                    int page_size, int n_pages, float scale, float *out,
                                    void *workspace, size_t workspace_bytes, int32_t *status,
                                    cudaStream_t stream) {
    if (!block_table || !k_scale || !v_scale) return GQA_ERR_NULL;
    if (!aligned(block_table, 4)) return GQA_ERR_ALIGNMENT;
    if (max_pages <= 0 || n_pages <= 0 || page_size <= 0 || page_size % 8 != 0 ||
        static_cast<long long>(max_pages) * page_size > (1ll << 30))
        return GQA_ERR_SHAPE;
    // a tile (256 or 128 rows) must lie in one page or cover whole pages
    if (256 % page_size != 0 && page_size % 256 != 0) return GQA_ERR_SHAPE;
    PagedArgs pg;
    pg.block_table = block_table;
    pg.max_pages = max_pages;
    pg.page_size = page_size;
    pg.n_pages = n_pages;
    return decode_impl(q, k_pool, v_pool, seq_lens, B, H_q, H_kv, d, max_pages * page_size, 0,
                       scale, GQA_DTYPE_E4M3, out, workspace, workspace_bytes, status, stream,
                       pg, 1, k_scale, v_scale);
}

extern "C" const char *gqa_status_string(int code) {
    switch (code) {
        case GQA_OK: return "ok";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_SHAPE: return "a size is not positive, too large, or not representable";
        case GQA_ERR_HEADS_NOT_DIVISIBLE: return "H_q is not a multiple of H_kv";
        case GQA_ERR_UNSUPPORTED_DIM: return "head dimension d must be 64 or 128";
        case GQA_ERR_UNSUPPORTED_DTYPE: return "unsupported element type";
        case GQA_ERR_ALIGNMENT: return "a pointer is not aligned as required";
        case GQA_ERR_WORKSPACE: return "workspace is NULL or too small";
        case GQA_ERR_CUDA: return "a CUDA runtime call failed";
        case GQA_ERR_NO_DEVICE: return "no usable sm_100 device is current";
        case GQA_ERR_SCRATCH_LIMIT: return "sizes need more scratch than the library's fixed no-allocation array";
        case GQA_ERR_OVERLAP: return "the input and output length arrays overlap";
        default: return "unknown status code";
    }
}

extern "C" int gqa_set_wait_timeout_ns(unsigned long long ns) {
    g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns);
    return GQA_OK;
}

extern "C" int gqa_profile_events(cudaEvent_t before_split, cudaEvent_t after_split) {
    g_ev_before.store(before_split);
    g_ev_after.store(after_split);
    return GQA_OK;
}
