// Log-sum-exp combine of split-KV partial results.
//
// A piece c of a unit holds, per query head, the unnormalised sum o_c = sum_t 2^(x_t - m_c) v_t,
// its reference m_c (log2 units) and l_c = sum_t 2^(x_t - m_c).  Because softmax is a ratio of
// sums of exponentials, the pieces merge exactly:
//     M = max_c m_c,   out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
// The pages state the blockwise idea (split the sequence into blocks, compute each block
// independently, then merge: "GQA注意力机制", section 4.2); the merge rule is the softmax
// algebra above.  Units covered by a single piece were finished by the split kernel and are
// skipped; units with no rows get zeros.
#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {

constexpr int kCombineThreads = 256;
constexpr int kCombineOutputsPerCta = 4 * kCombineThreads;

// grid = (units, chunks of kCombineOutputsPerCta outputs of one unit)
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const DecodeParams p) {
    extern __shared__ float csm[];
    int *piece_cta = reinterpret_cast<int *>(csm);  // CTA index of each piece, in line order
    float *wts = csm + p.G;                         // [piece][head] merge weight
    float *mref = wts + static_cast<long long>(p.G) * p.RB;  // [piece][head] reference max
    __shared__ int s_pieces;
    grid_dependency_wait();
    const int u = blockIdx.x;
    const int b = u / p.UB;
    const int k = u - b * p.UB;
    const int kvh = k / p.HB;
    const int hb = k - kvh * p.HB;
    const int nh = p.RB;  // columns of the unit (and slot layout stride)
    const int d = p.d;
    const int first = blockIdx.y * kCombineOutputsPerCta;
    const int last = min(nh * d, first + kCombineOutputsPerCta);
    if (first >= last) return;
    const long long *hdr = reinterpret_cast<const long long *>(p.ws);
    const int n = valid_len(p.seq_lens[b], p.L_max, p.Q);
    const int nt = seq_tiles(n, p);
    if (nt == 0) {
        for (int idx = first + threadIdx.x; idx < last; idx += blockDim.x) {
            const long long orow = out_row(p, b, kvh, hb, idx / d);
            if (orow >= 0) p.out[orow * d + idx % d] = 0.f;
        }
        return;
    }
    const long long total = hdr[p.B];
    const long long uoff = hdr[b] + static_cast<long long>(k) * nt;
    const int i0 = static_cast<int>(cta_of_tile(uoff, total, p.G));
    const int i1 = static_cast<int>(cta_of_tile(uoff + nt - 1, total, p.G));
    if (i0 == i1) return;  // one piece: the split kernel wrote the output
    // Every CTA in [i0, i1] holds a piece of this unit unless its range is empty, which can only
    // happen when there are fewer tiles than CTAs.
    if (total >= p.G) {
        for (int i = threadIdx.x; i <= i1 - i0; i += blockDim.x) piece_cta[i] = i0 + i;
        if (threadIdx.x == 0) s_pieces = i1 - i0 + 1;
    } else {
        for (int i = threadIdx.x; i <= i1 - i0; i += blockDim.x)
            piece_cta[i] = cta_range_begin(i0 + i, total, p.G) < cta_range_begin(i0 + i + 1, total, p.G) ? i0 + i : -1;
        __syncthreads();
        if (threadIdx.x == 0) {
            int c = 0;
            for (int i = 0; i <= i1 - i0; ++i)
                if (piece_cta[i] >= 0) piece_cta[c++] = piece_cta[i];
            s_pieces = c;
        }
    }
    __syncthreads();
    const int np = s_pieces;
    const float *slots = p.ws + p.hdr_floats + static_cast<long long>(u) * p.slot_floats;
    // weights: w[c][h] = 2^(m_c - M) / sum_c' 2^(m_c' - M) l_c'
    for (int idx = threadIdx.x; idx < np * nh; idx += blockDim.x) {
        const int c = idx / nh, h = idx - c * nh;
        const float *sl = slots + static_cast<long long>(piece_cta[c]) * p.slot_floats;
        mref[idx] = sl[nh * d + h];
        wts[idx] = sl[nh * d + nh + h];  // l_c for now
    }
    __syncthreads();
    for (int h = threadIdx.x; h < nh; h += blockDim.x) {
        float M = -INFINITY;
        for (int c = 0; c < np; ++c) M = fmaxf(M, mref[c * nh + h]);
        float den = 0.f;
        for (int c = 0; c < np; ++c) den = fmaf(ex2_approx(mref[c * nh + h] - M), wts[c * nh + h], den);
        const float inv = 1.f / den;
        for (int c = 0; c < np; ++c) wts[c * nh + h] = ex2_approx(mref[c * nh + h] - M) * inv;
    }
    __syncthreads();
    for (int idx = first + threadIdx.x; idx < last; idx += blockDim.x) {
        const int h = idx / d;
        const long long orow = out_row(p, b, kvh, hb, h);
        if (orow < 0) continue;
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < np; ++c)
            acc = fmaf(wts[c * nh + h], slots[static_cast<long long>(piece_cta[c]) * p.slot_floats + idx], acc);
        p.out[orow * d + (idx - h * d)] = acc;
    }
}

int launch_combine(const DecodeParams &p, cudaStream_t stream) {
    const long long units = static_cast<long long>(p.B) * p.UB;
    if (units == 0) return GQA_OK;
    const int chunks = (p.RB * p.d + kCombineOutputsPerCta - 1) / kCombineOutputsPerCta;
    const size_t smem = static_cast<size_t>(p.G) * (sizeof(int) + 2 * sizeof(float) * p.RB);
    static size_t smem_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    if (smem > 48 * 1024 && (dev >= 64 || smem_set[dev] < smem)) {
        if (cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return GQA_ERR_CUDA;
        if (dev < 64) smem_set[dev] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units), chunks);
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, combine_kernel, p) != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}

}  // namespace gqa
