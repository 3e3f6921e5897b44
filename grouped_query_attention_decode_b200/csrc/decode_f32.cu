// Split-KV GQA decode for float32 caches, on CUDA cores in float32.
//
// Same persistent partition as the tensor-core path (schedule.cuh), with 64-row tiles.  Per
// tile the CTA stages the group's K and V rows in shared memory once and serves all query
// heads of the group from them: scores (one (head, row) pair per thread), an online softmax per
// head (one warp per head), then the weighted sum of V (one (head, column) output per thread).
#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {

template <int D>
struct F32Cfg {
    static constexpr int T = 64;
    static constexpr int KP = D + 4;  // padded K row: conflict-free float4 row reads
    static constexpr int RBMAX = 64;
    static constexpr int SMEM_FLOATS = RBMAX * D + T * KP + T * D + RBMAX * T + 3 * RBMAX;
    static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
};

template <int D>
__global__ void __launch_bounds__(256)
split_f32_kernel(const float *__restrict__ q, const float *__restrict__ kc,
                 const float *__restrict__ vc, const DecodeParams p) {
    using C = F32Cfg<D>;
    constexpr int T = C::T;
    constexpr int KP = C::KP;
    extern __shared__ float4 fsm4[];
    float *const qs = reinterpret_cast<float *>(fsm4);  // [RBMAX][D]
    float *const ks = qs + C::RBMAX * D;                 // [T][KP]
    float *const vs = ks + T * KP;                       // [T][D]
    float *const ss = vs + T * D;                        // [RBMAX][T]
    float *const ms = ss + C::RBMAX * T;                 // running max per head (log2 units)
    float *const as = ms + C::RBMAX;                     // rescale factor of the last tile
    float *const ls = as + C::RBMAX;                     // running softmax denominator
    __shared__ long long s_begin, s_end, s_off0, s_offl, s_total;
    __shared__ int s_flag;
    __shared__ PendingPiece s_pend[2];
    __shared__ int s_b0, s_bl;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    grid_dependency_wait();
    if (warp == 0) {
        const CtaRange cr = locate_cta_range(p, blockIdx.x, lane, blockIdx.x == 0);
        if (lane == 0) {
            s_begin = cr.begin;
            s_end = cr.end;
            s_b0 = cr.b0;
            s_off0 = cr.off0;
            s_bl = cr.bl;
            s_offl = cr.offl;
            s_total = cr.total;
        }
    }
    __syncthreads();
    grid_launch_dependents();

    CtaRange cr;
    cr.begin = s_begin;
    cr.end = s_end;
    cr.b0 = s_b0;
    cr.off0 = s_off0;
    cr.bl = s_bl;
    cr.offl = s_offl;
    cr.total = s_total;
    SegmentWalker w;
    w.init(p, cr);
    Segment sg;
    PieceTickets tickets;
    int nseg = 0;
    zero_empty_units(p, blockIdx.x, tid, 256);  // units with no rows get zeros
    constexpr int ACC = C::RBMAX * D / 256;
    while (w.next(sg)) {
        // columns of the unit: (token j, head h') pairs, j * rb + h'
        const int nh = p.RB;
        for (int idx = tid; idx < nh * D; idx += 256) {
            const long long qr = out_row(p, sg.b, sg.kvh, sg.hb, idx / D);  // same row layout as out
            qs[idx] = qr >= 0 ? q[qr * D + idx % D] : 0.f;
        }
        if (tid < nh) {
            ms[tid] = -INFINITY;
            ls[tid] = 0.f;
        }
        float acc[ACC];
#pragma unroll
        for (int k = 0; k < ACC; ++k) acc[k] = 0.f;
        __syncthreads();
        for (int jj = 0; jj < sg.len; ++jj) {
            const int row0 = sg.first + sg.tile(jj) * T;
            const int rows = min(T, sg.n - row0);
            for (int idx = tid; idx < rows * (D / 4); idx += 256) {
                const int t = idx / (D / 4);
                const int c4 = idx - t * (D / 4);
                // element offset of cached row row0 + t of this key/value head
                long long off;
                if (p.block_table != nullptr) {
                    const int lr = row0 + t;
                    int pg = p.block_table[static_cast<long long>(sg.b) * p.max_pages + lr / p.page_size];
                    if (pg < 0 || pg >= p.n_pages) {
                        if (p.status != nullptr) atomicOr(p.status, GQA_STATUS_PAGE_RANGE);
                        pg = 0;
                    }
                    off = ((static_cast<long long>(pg) * p.page_size + lr % p.page_size) * p.H_kv + sg.kvh) * D;
                } else {
                    off = ((static_cast<long long>(sg.b) * p.L_max + row0 + t) * p.H_kv + sg.kvh) * D;
                }
                const float4 kv = *reinterpret_cast<const float4 *>(kc + off + 4 * c4);
                const float4 vv = *reinterpret_cast<const float4 *>(vc + off + 4 * c4);
                *reinterpret_cast<float4 *>(ks + t * KP + 4 * c4) = kv;
                *reinterpret_cast<float4 *>(vs + t * D + 4 * c4) = vv;
            }
            __syncthreads();
            for (int idx = tid; idx < nh * T; idx += 256) {
                const int h = idx / T;
                const int t = idx - h * T;
                float s = -INFINITY;
                // token j = h / rb of the unit sees rows < n - Q + 1 + j
                if (t < rows && row0 + t < sg.n - p.Q + 1 + h / p.rb) {
                    const float4 *qa = reinterpret_cast<const float4 *>(qs + h * D);
                    const float4 *ka = reinterpret_cast<const float4 *>(ks + t * KP);
                    float a = 0.f;
#pragma unroll 8
                    for (int c = 0; c < D / 4; ++c) {
                        const float4 x = qa[c], y = ka[c];
                        a = fmaf(x.x, y.x, a);
                        a = fmaf(x.y, y.y, a);
                        a = fmaf(x.z, y.z, a);
                        a = fmaf(x.w, y.w, a);
                    }
                    s = a * p.scale_log2;
                }
                ss[h * T + t] = s;
            }
            __syncthreads();
            for (int h = warp; h < nh; h += 8) {
                const float a = ss[h * T + lane], b = ss[h * T + lane + 32];
                const float tmax = warp_max_f32(fmaxf(a, b));
                const float m_old = ms[h];
                const float m_new = fmaxf(m_old, tmax);
                // no visible row yet (several query tokens): nothing to rescale or add
                const bool none = m_new == -INFINITY;
                const float alpha = none ? 1.f : ex2_approx(m_old - m_new);
                const float pa = a == -INFINITY ? 0.f : ex2_approx(a - m_new);
                const float pb = b == -INFINITY ? 0.f : ex2_approx(b - m_new);
                ss[h * T + lane] = pa;
                ss[h * T + lane + 32] = pb;
                const float sum = warp_sum_f32(pa + pb);
                if (lane == 0) {
                    ls[h] = ls[h] * alpha + sum;
                    ms[h] = m_new;
                    as[h] = alpha;
                }
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < ACC; ++k) {
                const int idx = tid + 256 * k;
                if (idx < nh * D) {
                    const int h = idx / D;
                    const int c = idx - h * D;
                    float a = acc[k] * as[h];
                    const float *pr = ss + h * T;
                    for (int t = 0; t < rows; ++t) a = fmaf(pr[t], vs[t * D + c], a);
                    acc[k] = a;
                }
            }
            __syncthreads();
        }
        if (sg.whole) {
#pragma unroll
            for (int k = 0; k < ACC; ++k) {
                const int idx = tid + 256 * k;
                if (idx < nh * D) {
                    const long long orow = out_row(p, sg.b, sg.kvh, sg.hb, idx / D);
                    if (orow >= 0) p.out[orow * D + idx % D] = acc[k] / ls[idx / D];
                }
            }
        } else {
            float *slot = p.ws + p.slot_base + (static_cast<long long>(blockIdx.x) + sg.unit) * p.slot_floats;
#pragma unroll
            for (int k = 0; k < ACC; ++k) {
                const int idx = tid + 256 * k;
                if (idx < nh * D) slot[idx] = acc[k];
            }
            if (tid < nh) {
                slot[nh * D + tid] = ms[tid];
                slot[nh * D + nh + tid] = ls[tid];
            }
        }
        __syncthreads();
        if (!sg.whole) tickets.record(p, sg, 0, tid, s_pend);
        // the range's partial pieces come first: merge what they complete right away
        if (++nseg == 2) tickets.finish(p, cr.total, 0, 0, p.RB, tid, 256, s_pend, &s_flag, [] { __syncthreads(); });
    }
    // units cut into pieces are merged by the CTA holding the last ticket
    tickets.finish(p, cr.total, 0, 0, p.RB, tid, 256, s_pend, &s_flag, [] { __syncthreads(); });
}

template <int D>
static int launch_split_f32_impl(const DecodeParams &p, const float *q, const float *kc,
                                 const float *vc, cudaStream_t stream) {
    using C = F32Cfg<D>;
    auto kern = split_f32_kernel<D>;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return GQA_ERR_CUDA;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.G);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, q, kc, vc, p) != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}

int launch_split_f32(const DecodeParams &p, const float *q, const float *kc, const float *vc,
                     cudaStream_t stream) {
    if (p.d == 128) return launch_split_f32_impl<128>(p, q, kc, vc, stream);
    return launch_split_f32_impl<64>(p, q, kc, vc, stream);
}

}  // namespace gqa
