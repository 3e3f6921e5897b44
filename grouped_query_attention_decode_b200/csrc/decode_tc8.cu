// Split-KV GQA decode over an FP8 (e4m3) KV cache with one scale per key/value head, on
// sm_100a tensor cores (tcgen05 kind::f8f6f4 + TMA).
//
// "GQA 阅读笔记", section "复现性与工程实践", mixed-precision item: serving systems keep the KV
// cache in FP8, which halves GQA's per-step KV bytes again.  A stored code c of key/value head
// g stands for value(c) * k_scale[g] (K) or value(c) * v_scale[g] (V).  The codes go to the
// tensor cores as they are, straight from the TMA ring; the scales act outside the products:
//
//   S^T[T rows x 2RP] = K_codes[T x d] . [q_hi | q_lo]^T              (UMMA, M=128 per half)
//   score_h  = (S_hi + S_lo / 16) * k_scale[g] * softmax scale / c_h
//   O^T[d x 3RP]     = V_codes^T[d x T] . [P_hi | P_mid | P_lo]^T     (UMMA, M=d, K=T)
//   O_h += O_hi + O_mid / 16 + O_lo / 256;    out = O * v_scale[g] / l
//
// q (bf16) becomes two e4m3 terms after each query row is multiplied by a power of two c_h
// that puts its largest magnitude in [128, 256): q*c_h = q_hi + q_lo/16 holds the bf16 value
// exactly for every element within 2^10 of the row's largest.  The softmax numerators
// P = 2^(s - m) <= 2^8 (lazy rescale) become three e4m3 terms 16x apart: ~12 significant bits
// for P >= 2^-6, and an absolute error below 2^-18 under that.  Both products put their terms
// side by side along N, so each K and V tile is read from shared memory once per product.
//
// A tile is T = 256 rows (NH <= 16 heads per unit) or 128 rows, so that one K+V stage of a
// d = 128 cache is 64 KB or 32 KB.  Roles, barriers, the lazy rescale, the bounded waits and
// the drain on abort follow the bf16 kernel (decode_tc.cu); the differences are the e4m3
// operands, the q conversion -- done by the producer warp from global memory, once per unit --
// and the three-term P.
#include <cuda_bf16.h>

#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {
namespace {

constexpr unsigned long long kDrainNs8 = 1000000000ull;
constexpr float kLazyLog2_8 = 8.0f;  // P <= 2^8 = 256 stays inside e4m3's range (448)

template <int D, int NH>
struct Tc8Cfg {
    static constexpr int RP = NH < 16 ? 16 : NH;       // query columns per term (UMMA N / 2)
    static constexpr int T = NH <= 16 ? 256 : 128;     // tile rows
    static constexpr int RT = T / 128;                 // tile rows per softmax thread
    static constexpr int ROWB = D;                     // bytes of a cached row
    static constexpr uint32_t KV_LAYOUT = D == 128 ? 2u : 4u;  // 128- / 64-byte swizzle
    static constexpr int TILE_BYTES = T * ROWB;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int Q8_BYTES = 2 * RP * ROWB;     // rows [q_hi of RP columns | q_lo]
    // P^T: three e4m3 terms, each MN-major [T rows][RP bytes]; a row of 16 / 32 / 64 bytes is
    // laid out without swizzle / with 32-byte / with 64-byte swizzle.  The terms are the three
    // MN blocks of one N = 3*RP operand.
    static constexpr int P_TERM = T * RP;
    static constexpr int P_BYTES = 3 * P_TERM;
    static constexpr uint32_t P_LAYOUT = RP == 16 ? 0u : RP == 32 ? 6u : 4u;
    //   no swizzle: core matrices of 16 bytes x 8 rows; MN blocks SBO apart, 8-row groups LBO
    //   swizzled:   MN atoms LBO apart, 8-row groups SBO apart
    static constexpr uint32_t P_LBO = RP == 16 ? 128u : static_cast<uint32_t>(P_TERM);
    static constexpr uint32_t P_SBO = RP == 16 ? static_cast<uint32_t>(P_TERM) : 8u * RP;
    // TMEM: S^T (2 buffers x RT row halves x 2RP), then O^T (OB buffers x 3RP)
    static constexpr int S_COLS = 2 * RT * 2 * RP;
    static constexpr int OB = S_COLS + 2 * 3 * RP <= 512 ? 2 : 1;
    static constexpr int O_COL = S_COLS;
    static constexpr int USED = S_COLS + OB * 3 * RP;
    static constexpr int TMEM_COLS = USED <= 128 ? 128 : (USED <= 256 ? 256 : 512);
    static constexpr uint32_t IDESC_QK = idesc_e4m3_f32(128, 2 * RP, false, false);
    static constexpr uint32_t IDESC_PV = idesc_e4m3_f32(D, 3 * RP, true, true);
    static constexpr int NWG = NH >= 32 ? NH / 16 : 1;
    static constexpr int NHW = NH / NWG;
    // 256-row tiles: one warpgroup per 128-row half, so every softmax thread owns one row and
    // a tile's softmax takes the time of 128 rows
    static constexpr int RS = RT;
    static constexpr int NSW = NWG * RS;               // softmax warpgroups
    static constexpr int TICKET_WARP = 2 + 4 * NSW;    // the ticket warp (schedule.cuh)
    static constexpr int THREADS = 64 + 128 * NSW + 32;
    static constexpr int NHW4 = (NHW + 3) / 4;
    static constexpr int LOG2NHW = NHW >= 16 ? 4 : NHW >= 8 ? 3 : NHW >= 4 ? 2 : NHW >= 2 ? 1 : 0;

    struct Small {
        // K and V of a stage land on separate barriers: S = K.Q^T starts as soon as K is in,
        // while V is still on its way; the stage is released after P.V
        uint64_t k_full[8], v_full[8], kv_empty[8];
        uint64_t q_full[2], q_empty[2], qf_empty[2];
        uint64_t s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2];
        uint64_t mma_done;
        uint64_t pc_full[kPieceGroups][2];  // a group's partial piece is in its slot
        uint64_t tk_done[kPieceGroups][2];  // its ticket is taken: tk_last says if it was the last
        int tk_last[kPieceGroups][2];  // a head slice's partial piece is in its slot
        uint32_t tmem_base;
        int abort;
        int b0, bl;
        long long begin, end, off0, offl, total;
        float qf[2][RP];                    // score factor of each column: scale * k_scale / c_h
        float vsc[2];                       // v_scale of the unit's key/value head
        float4 wmax[NWG][2][4 * RS][NHW4];  // per head slice, S buffer, warp: warp maxima
        float lsum[NWG][4 * RS][NHW];
    };

    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int BASE = 2 * P_BYTES + static_cast<int>((sizeof(Small) + 1023) / 1024 * 1024);
    static constexpr int QB = (SMEM_LIMIT - BASE - 2 * Q8_BYTES >= 2 * STAGE_BYTES) ? 2 : 1;
    static constexpr int FIXED = BASE + QB * Q8_BYTES;
    static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE_BYTES;
    static constexpr int S = S_FIT > 8 ? 8 : S_FIT;
    static constexpr int SMEM_BYTES = S * STAGE_BYTES + FIXED;
    static_assert(S >= 2, "shared memory too small for a double-buffered ring");
    static_assert(!(D == 128 && T == 256) || S >= 3, "64 KB stages: keep three in the ring");
    static_assert(RS == 1 || NWG == 1, "row halves split only with one head slice");
    static_assert(Q8_BYTES % 1024 == 0 && P_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "");
};

template <int NH, int LOG2NH>
__device__ __forceinline__ void warp_max_transpose8(float (&v)[NH], int lane) {
#pragma unroll
    for (int s = 0; s < LOG2NH; ++s) {
        const int half = NH >> (s + 1);
        const bool upper = (lane >> s) & 1;
#pragma unroll
        for (int j = 0; j < NH / 2; ++j) {
            if (j < half) {
                const float send = upper ? v[j] : v[j + half];
                const float keep = upper ? v[j + half] : v[j];
                v[j] = fmaxf(keep, __shfl_xor_sync(kFullMask, send, 1 << s));
            }
        }
    }
#pragma unroll
    for (int off = 1 << LOG2NH; off < 32; off <<= 1) v[0] = fmaxf(v[0], __shfl_xor_sync(kFullMask, v[0], off));
}

template <int NH, int LOG2NH>
__device__ __forceinline__ int transpose_head8(int lane) {
    int h = 0;
#pragma unroll
    for (int s = 0; s < LOG2NH; ++s) h += ((lane >> s) & 1) * (NH >> (s + 1));
    return h;
}

__device__ __forceinline__ uint64_t desc_add8(uint64_t desc, uint32_t bytes) {
    return desc + static_cast<uint64_t>(bytes >> 4);
}

// Byte offset of 16-byte chunk `c` of row `r` in a K-major tile of `rowb`-byte rows with the
// 128-byte (rowb = 128) or 64-byte (rowb = 64) swizzle the TMA and the UMMA descriptors use.
template <int ROWB>
__device__ __forceinline__ uint32_t kmajor_chunk(int r, int c) {
    const int x = ROWB == 128 ? (r & 7) : ((r >> 1) & 3);
    return static_cast<uint32_t>(r * ROWB + ((c ^ x) << 4));
}

// Byte offset of the 16-byte chunk `c` of row `t` of one MN-major P^T term.
template <int RP>
__device__ __forceinline__ uint32_t p_chunk(int t, int c) {
    const int x = RP == 16 ? 0 : RP == 32 ? ((t >> 2) & 1) : ((t >> 1) & 3);
    return static_cast<uint32_t>(t * RP + ((c ^ x) << 4));
}

// One pair of P values split into three e4m3 terms 16x apart: p = hi + mid/16 + lo/256 to
// ~12 significant bits.  The pair is first rounded to f16 (11 bits); each residual is exact in
// f16 before its scaling by 16.
__device__ __forceinline__ void split3(float a, float b, uint16_t &hi, uint16_t &mid, uint16_t &lo) {
    const uint32_t sixteen = 0x4C004C00u;  // f16x2 {16, 16}
    const uint32_t h = f16x2_from_f32(a, b);
    hi = e4m3x2_from_f16x2(h);
    const uint32_t r1 = f16x2_mul(f16x2_sub(h, f16x2_from_e4m3x2(hi)), sixteen);
    mid = e4m3x2_from_f16x2(r1);
    const uint32_t r2 = f16x2_mul(f16x2_sub(r1, f16x2_from_e4m3x2(mid)), sixteen);
    lo = e4m3x2_from_f16x2(r2);
}

template <int D, int NH, bool PAGED>
__global__ void __launch_bounds__(Tc8Cfg<D, NH>::THREADS, 1)
split_tc8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_k8,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_v8,
                 const __nv_bfloat16 *__restrict__ q, const DecodeParams p) {
    using C = Tc8Cfg<D, NH>;
    constexpr int T = C::T;
    constexpr int S = C::S;
    constexpr int RP = C::RP;
    constexpr int RT = C::RT;
    constexpr int ROWB = C::ROWB;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *const st_base = smem;
    uint8_t *const q8_base = smem + S * C::STAGE_BYTES;
    uint8_t *const p_base = q8_base + C::QB * C::Q8_BYTES;
    auto *const sm = reinterpret_cast<typename C::Small *>(p_base + 2 * C::P_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0 && p.status != nullptr) atomicOr(p.status, GQA_STATUS_INTERNAL);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&sm->k_full[s], 1);
            mbar_init(&sm->v_full[s], 1);
            mbar_init(&sm->kv_empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm->q_full[j], 1);
            mbar_init(&sm->q_empty[j], 1);               // the unit's last S^T has been computed
            mbar_init(&sm->qf_empty[j], 4 * C::NSW);    // every softmax warp read the factors
            mbar_init(&sm->s_full[j], 1);
            mbar_init(&sm->s_empty[j], 4 * C::NSW);
            mbar_init(&sm->p_full[j], 4 * C::NSW);
            mbar_init(&sm->o_full[j], 1);
            mbar_init(&sm->o_empty[j], 4 * C::NWG);     // the first row half folds O
        }
        mbar_init(&sm->mma_done, 1);
        for (int g = 0; g < kPieceGroups; ++g) {
            mbar_init(&sm->pc_full[g][0], 1);
            mbar_init(&sm->pc_full[g][1], 1);
            mbar_init(&sm->tk_done[g][0], 1);
            mbar_init(&sm->tk_done[g][1], 1);
        }
        sm->abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_k8);
        prefetch_tmap(&tm_v8);
    }
    // Everything below reads what the previous kernel on the stream (the append) wrote.
    grid_dependency_wait();
    if (warp == 2) {
        const CtaRange cr = locate_cta_range(p, blockIdx.x, lane, blockIdx.x == 0);
        if (lane == 0) {
            sm->begin = cr.begin;
            sm->end = cr.end;
            sm->b0 = cr.b0;
            sm->off0 = cr.off0;
            sm->bl = cr.bl;
            sm->offl = cr.offl;
            sm->total = cr.total;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    grid_launch_dependents();

    const uint32_t tmem = sm->tmem_base;
    CtaRange cr;
    cr.begin = sm->begin;
    cr.end = sm->end;
    cr.b0 = sm->b0;
    cr.off0 = sm->off0;
    cr.bl = sm->bl;
    cr.offl = sm->offl;
    cr.total = sm->total;
    volatile int *abort_flag = &sm->abort;
    const uint64_t budget = p.wait_ns;

    auto fail = [&]() {
        *abort_flag = 1;
        if (p.status != nullptr) atomicOr(p.status, GQA_STATUS_WAIT_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------------ producer warp
        // Walks the tile line with all 32 lanes.  Per unit it converts q into the e4m3 operand
        // (below); per tile lane 0 waits for a free stage and the copies are issued one box per
        // lane (a paged cache: each lane owns one page-sized box, whose page id it loaded
        // kPageAhead tiles earlier).
        const uint64_t pol = l2_policy_evict_first();
        SegmentWalker w;
        w.init(p, cr);
        Segment sg;
        int i = 0, sidx = 0;
        bool ok = true;
        [[maybe_unused]] TileCursor ahead;
        [[maybe_unused]] int pg_ring[kPageAhead];
        if constexpr (PAGED) {
            ahead.init(p, cr);
#pragma unroll
            for (int k = 0; k < kPageAhead; ++k) {
                pg_ring[k] = ahead.page_of_box(p, T, lane);
                ahead.advance();
            }
        }
        // q of the current unit -> rows [q_hi | q_lo] of the unit's q buffer (K-major, swizzled
        // like the cache tiles) and 1/c_h per column.  8 lanes per q row, D/8 elements each.
        auto convert_q = [&](int qb, const Segment &su) {
            constexpr int V = D / 8;
            uint8_t *q8 = q8_base + qb * C::Q8_BYTES;
            const int sub = lane >> 3, seg = lane & 7;
            const float kfac = p.scale_log2 * p.k_scale[su.kvh];
            if (lane == 0) sm->vsc[qb] = p.v_scale[su.kvh];
#pragma unroll 1
            for (int r0 = 0; r0 < RP; r0 += 4) {
                const int rr = r0 + sub;
                const long long qrow = rr < p.RB ? out_row(p, su.b, su.kvh, su.hb, rr) : -1;
                float v[V];
                if (qrow >= 0) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(q + qrow * D + seg * V);
#pragma unroll
                    for (int u = 0; u < V / 8; ++u) {
                        const uint4 raw = src[u];
                        const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[u * 8 + 2 * k] = __uint_as_float(wds[k] << 16);
                            v[u * 8 + 2 * k + 1] = __uint_as_float(wds[k] & 0xFFFF0000u);
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < V; ++k) v[k] = 0.f;
                }
                float mx = 0.f;
#pragma unroll
                for (int k = 0; k < V; ++k) mx = fmaxf(mx, fabsf(v[k]));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 4));
                // c = 2^(7 - floor(log2 mx)), so that mx * c lies in [128, 256)
                const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
                int sh = 7 - e;
                sh = sh < -120 ? -120 : (sh > 120 ? 120 : sh);
                const float c = __uint_as_float(static_cast<uint32_t>(127 + sh) << 23);
                uint32_t hw[V / 4], lw[V / 4];
#pragma unroll
                for (int k = 0; k < V; k += 4) {
                    uint16_t h2[2], l2[2];
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const float a = v[k + 2 * k2] * c, b = v[k + 2 * k2 + 1] * c;
                        h2[k2] = e4m3x2_from_f32(a, b);
                        const float2 back = f32x2_from_f16x2(f16x2_from_e4m3x2(h2[k2]));
                        l2[k2] = e4m3x2_from_f32((a - back.x) * 16.f, (b - back.y) * 16.f);
                    }
                    hw[k / 4] = static_cast<uint32_t>(h2[0]) | (static_cast<uint32_t>(h2[1]) << 16);
                    lw[k / 4] = static_cast<uint32_t>(l2[0]) | (static_cast<uint32_t>(l2[1]) << 16);
                }
                if constexpr (V == 16) {
                    *reinterpret_cast<uint4 *>(q8 + kmajor_chunk<ROWB>(rr, seg)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(q8 + kmajor_chunk<ROWB>(RP + rr, seg)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                } else {
                    const uint32_t half = (seg & 1) * 8;
                    *reinterpret_cast<uint2 *>(q8 + kmajor_chunk<ROWB>(rr, seg >> 1) + half) = make_uint2(hw[0], hw[1]);
                    *reinterpret_cast<uint2 *>(q8 + kmajor_chunk<ROWB>(RP + rr, seg >> 1) + half) = make_uint2(lw[0], lw[1]);
                }
                if (seg == 0) sm->qf[qb][rr] = kfac * __uint_as_float(static_cast<uint32_t>(127 - sh) << 23);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->q_full[qb]);
        };
        while (ok && w.next(sg)) {
            const int qb = sidx % C::QB;
            bool got = true;
            if (lane == 0 && sidx >= C::QB)
                got = wait_bounded(&sm->q_empty[qb], ((sidx / C::QB) - 1) & 1, abort_flag, budget) &&
                      wait_bounded(&sm->qf_empty[qb], ((sidx / C::QB) - 1) & 1, abort_flag, budget);
            if (!__shfl_sync(kFullMask, got, 0)) {
                ok = false;
                break;
            }
            ++sidx;
            // The conversion waits on global loads.  The CTA's first unit converts before any
            // tile is requested (its loads would otherwise queue behind every CTA's first
            // stages); later units convert when the ring is full (before the first wait for a
            // free stage), or once their tiles are all issued.
            bool q_pending = true;
            if (i == 0) {
                convert_q(qb, sg);
                q_pending = false;
            }
            for (int jj = 0; jj < sg.len; ++jj) {
                const int st = i % S;
                const int row0 = sg.first + sg.tile(jj) * T;
                const int rows = min(T, sg.n - row0);
                [[maybe_unused]] int pg = 0;
                if constexpr (PAGED) {
                    pg = pg_ring[0];
#pragma unroll
                    for (int k = 0; k + 1 < kPageAhead; ++k) pg_ring[k] = pg_ring[k + 1];
                    pg_ring[kPageAhead - 1] = ahead.page_of_box(p, T, lane);
                    ahead.advance();
                }
                if (q_pending && i >= S) {
                    convert_q(qb, sg);
                    q_pending = false;
                }
                got = true;
                if (lane == 0 && i >= S)
                    got = wait_bounded(&sm->kv_empty[st], ((i / S) - 1) & 1, abort_flag, budget);
                if (!__shfl_sync(kFullMask, got, 0)) {
                    ok = false;
                    break;
                }
                uint8_t *kdst = st_base + st * C::STAGE_BYTES;
                uint8_t *vdst = kdst + C::TILE_BYTES;
                // boxes: the whole tile, pages of min(page_size, T) rows, or 8-row boxes for a
                // partial tile (at most 7 rows past n)
                int boxr, nbox;
                if constexpr (PAGED) {
                    boxr = rows == T ? min(p.page_size, T) : 8;
                    nbox = rows == T ? T / boxr : (rows + 7) >> 3;
                } else {
                    boxr = rows == T ? T : 8;
                    nbox = rows == T ? 1 : (rows + 7) >> 3;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm->k_full[st], nbox * boxr * ROWB);
                    mbar_arrive_expect_tx(&sm->v_full[st], nbox * boxr * ROWB);
                }
                __syncwarp();
                if (lane < nbox) {
                    const CUtensorMap *mk = rows == T ? &tm_k : &tm_k8;
                    const CUtensorMap *mv = rows == T ? &tm_v : &tm_v8;
                    const uint32_t off = lane * boxr * ROWB;
                    if constexpr (PAGED) {
                        if (pg < 0 || pg >= p.n_pages) {
                            if (p.status != nullptr) atomicOr(p.status, GQA_STATUS_PAGE_RANGE);
                            pg = 0;
                        }
                        const int pr = (row0 + lane * boxr) % p.page_size;
                        tma_load_4d(kdst + off, mk, &sm->k_full[st], 0, sg.kvh, pr, pg, pol);
                        tma_load_4d(vdst + off, mv, &sm->v_full[st], 0, sg.kvh, pr, pg, pol);
                    } else {
                        tma_load_4d(kdst + off, mk, &sm->k_full[st], 0, sg.kvh, row0 + lane * boxr, sg.b, pol);
                        tma_load_4d(vdst + off, mv, &sm->v_full[st], 0, sg.kvh, row0 + lane * boxr, sg.b, pol);
                    }
                }
                ++i;
            }
            if (ok && q_pending) convert_q(qb, sg);
        }
        if (lane == 0) {
            if (!ok) fail();
            for (int ii = (i > S ? i - S : 0); ii < i; ++ii) {
                wait_bounded(&sm->k_full[ii % S], (ii / S) & 1, nullptr, kDrainNs8);
                wait_bounded(&sm->v_full[ii % S], (ii / S) & 1, nullptr, kDrainNs8);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            // K tile, [q_hi | q_lo]: K-major, 8-row groups 8*ROWB apart.  V^T: MN-major, one
            // atom along d.  P^T: MN-major, three term blocks along N.
            const uint64_t dk0 = sdesc_swz(smem_u32(st_base), 16, 8 * ROWB, C::KV_LAYOUT);
            const uint64_t dv0 = sdesc_swz(smem_u32(st_base + C::TILE_BYTES), C::TILE_BYTES, 8 * ROWB, C::KV_LAYOUT);
            const uint64_t dq0 = sdesc_swz(smem_u32(q8_base), 16, 8 * ROWB, C::KV_LAYOUT);
            const uint64_t dp0 = sdesc_swz(smem_u32(p_base), C::P_LBO, C::P_SBO, C::P_LAYOUT);
            SegmentWalker w;
            w.init(p, cr);
            Segment sg;
            bool qk_more = w.next(sg);
            int qk_t = 0, qk_jj = 0, sidx = 0, pv_t = 0;
            bool q_ready = false;
            bool ok = true;
            uint64_t idle_since = global_timer_ns();
            uint32_t idle_polls = 0;
            while (qk_more || pv_t < qk_t) {
                bool progress = false;
                // P.V first: it is what releases a stage, so it never waits behind the next
                // tile's S^T.
                if (pv_t < qk_t) {
                    const int j2 = pv_t & 1;
                    const int ob = pv_t % C::OB;
                    if (mbar_test_wait(&sm->p_full[j2], (pv_t >> 1) & 1) &&
                        mbar_test_wait(&sm->v_full[pv_t % S], (pv_t / S) & 1) &&
                        (pv_t < C::OB || mbar_test_wait(&sm->o_empty[ob], ((pv_t / C::OB) - 1) & 1))) {
                        tc_fence_after_sync();
                        const uint64_t dv = desc_add8(dv0, (pv_t % S) * C::STAGE_BYTES);
                        const uint64_t dp = desc_add8(dp0, j2 * C::P_BYTES);
#pragma unroll
                        for (int kk = 0; kk < T / 32; ++kk) {
                            umma_f8(tmem + C::O_COL + ob * 3 * RP, desc_add8(dv, kk * 32 * ROWB),
                                    desc_add8(dp, kk * 32 * RP), C::IDESC_PV, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&sm->o_full[ob]);
                        umma_commit(&sm->kv_empty[pv_t % S]);
                        ++pv_t;
                        progress = true;
                    }
                }
                if (qk_more) {
                    const int qb = sidx % C::QB;
                    if (!q_ready) q_ready = mbar_test_wait(&sm->q_full[qb], (sidx / C::QB) & 1);
                    const int st = qk_t % S;
                    const int j2 = qk_t & 1;
                    if (q_ready && mbar_test_wait(&sm->k_full[st], (qk_t / S) & 1) &&
                        (qk_t < 2 || mbar_test_wait(&sm->s_empty[j2], ((qk_t >> 1) - 1) & 1))) {
                        tc_fence_after_sync();
                        const uint64_t dk = desc_add8(dk0, st * C::STAGE_BYTES);
                        const uint64_t dq = desc_add8(dq0, qb * C::Q8_BYTES);
#pragma unroll
                        for (int hf = 0; hf < RT; ++hf) {
#pragma unroll
                            for (int kk = 0; kk < D / 32; ++kk) {
                                umma_f8(tmem + (j2 * RT + hf) * 2 * RP, desc_add8(dk, hf * 128 * ROWB + kk * 32),
                                        desc_add8(dq, kk * 32), C::IDESC_QK, kk > 0 ? 1u : 0u);
                            }
                        }
                        umma_commit(&sm->s_full[j2]);
                        ++qk_t;
                        if (++qk_jj == sg.len) {
                            umma_commit(&sm->q_empty[qb]);
                            ++sidx;
                            qk_jj = 0;
                            q_ready = false;
                            qk_more = w.next(sg);
                        }
                        progress = true;
                    }
                }
                if (progress) {
                    idle_polls = 0;
                } else if ((++idle_polls & 15u) == 0) {
                    if (idle_polls == 16) idle_since = global_timer_ns();
                    if (*abort_flag || global_timer_ns() - idle_since > budget) {
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) fail();
            umma_commit(&sm->mma_done);
            wait_bounded(&sm->mma_done, 0, nullptr, kDrainNs8);
        }
    } else if (warp == C::TICKET_WARP) {
        // ------------------------------------------------------------------ ticket warp
        run_ticket_warp<C::NWG>(p, cr, sm->pc_full, sm->tk_done, sm->tk_last, lane, abort_flag, budget);
    } else {
        // ------------------------------------------------------------------ softmax warps
        // Every softmax thread owns one row of each tile.  NWG warpgroups split the heads
        // (NH >= 32, 128-row tiles), or -- 256-row tiles -- RS = 2 warpgroups split the rows:
        // warpgroup w takes rows [128w, 128w + 128) of every tile.  The two halves share the
        // running maximum (the warp maxima of both are exchanged) and the row sums; the first
        // half folds the Oᵀ tiles into registers and writes the result.
        constexpr int NHW = C::NHW;
        constexpr int RS = C::RS;
        constexpr int SCOLS = C::NWG == 1 ? RP : NHW;
        constexpr int NBAR = 128 * RS;                // threads at the group's named barrier
        const int wgi = (warp - 2) >> 2;              // 0 .. NSW - 1
        const int hf = RS == 2 ? wgi : 0;             // row half
        const int wg = RS == 2 ? 0 : wgi;             // head slice
        const bool folds = hf == 0;                   // folds O and writes the result
        const int hbase = wg * NHW;
        const uint32_t bar_id = 1 + wg;
        const int q4 = warp & 3;
        const int wq = hf * 4 + q4;                   // warp index within the group (0 .. 4RS-1)
        const int row = q4 * 32 + lane;               // row of the tile half (TMEM lane)
        const int trow = hf * 128 + row;              // row of the tile
        const int sm_tid = threadIdx.x - 64 - 128 * (RS == 2 ? 0 : wg);  // 0 .. NBAR-1 in the group
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int dcol = (D == 128) ? row : (lane < 16 ? q4 * 16 + lane : -1);
        SegmentWalker w;
        w.init(p, cr);
        Segment sg;
        int i = 0, sidx = 0;
        bool ok = true;
        float O[NHW], l[NHW], m_run[NHW], alpha[NHW], f[NHW];
        int npart = 0, nmerged = 0;  // partial pieces handed to the ticket warp, reports taken
        PendingPiece parts[2];
        auto merge_in = [&](bool block) {
            return merge_reported(p, cr.total, wg, hbase, hbase + NHW, sm_tid, NBAR, sm->tk_done[wg], sm->tk_last[wg],
                                  parts, npart, nmerged, block, abort_flag, budget,
                                  [&](bool pred) { return named_bar_any(bar_id, NBAR, pred); });
        };
        // units with no rows get zeros (while the first tiles are still on their way)
        zero_empty_units(p, blockIdx.x, threadIdx.x - 64, 128 * C::NSW);
        // O of tile t folded into the running sum, scaled by `scale_by` (first row half only)
        auto fold_o = [&](int t, const float *scale_by) -> bool {
            const int ob = t % C::OB;
            if (!wait_bounded(&sm->o_full[ob], (t / C::OB) & 1, abort_flag, budget)) return false;
            tc_fence_after_sync();
            const uint32_t obase = tmem + lane_addr + C::O_COL + ob * 3 * RP + hbase;
#pragma unroll
            for (int c = 0; c < NHW; c += 16) {
                uint32_t hi[16], mi[16], lo[16];
                tmem_ld16(obase + c, hi);
                tmem_ld16(obase + RP + c, mi);
                tmem_ld16(obase + 2 * RP + c, lo);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (c + e < NHW) {
                        const float o = __uint_as_float(hi[e]) + 0.0625f * __uint_as_float(mi[e]) +
                                        0.00390625f * __uint_as_float(lo[e]);
                        O[c + e] = scale_by != nullptr ? (O[c + e] + o) * scale_by[c + e] : O[c + e] + o;
                    }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->o_empty[ob]);
            return true;
        };
        while (ok && w.next(sg)) {
#pragma unroll
            for (int h = 0; h < NHW; ++h) {
                O[h] = 0.f;
                l[h] = 0.f;
                m_run[h] = -INFINITY;
            }
            bool bad = false;
            // The unit's score factors (softmax scale in log2 units * k_scale[g] / c_h) and
            // v_scale[g], written by the producer with the converted q.
            const int qb = sidx % C::QB;
            float vs = 0.f;
            if (wait_bounded(&sm->q_full[qb], (sidx / C::QB) & 1, abort_flag, budget)) {
#pragma unroll
                for (int h = 0; h < NHW; ++h) f[h] = sm->qf[qb][hbase + h];
                vs = sm->vsc[qb];
            } else {
                bad = true;
#pragma unroll
                for (int h = 0; h < NHW; ++h) f[h] = 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->qf_empty[qb]);
            ++sidx;
            for (int jj = 0; jj < sg.len; ++jj, ++i) {
                const int j2 = i & 1;
                const int rows = min(T, sg.n - sg.first - sg.tile(jj) * T);
                if (rows < T && !bad && wait_bounded(&sm->v_full[i % S], (i / S) & 1, abort_flag, budget)) {
                    // Rows past n: zero V so that 0-weight rows add exactly 0.
                    uint8_t *vbase = st_base + (i % S) * C::STAGE_BYTES + C::TILE_BYTES;
                    constexpr int CPR = ROWB / 16;
                    for (int c = sm_tid; c < (T - rows) * CPR; c += NBAR)
                        *reinterpret_cast<uint4 *>(vbase + (rows + c / CPR) * ROWB + (c % CPR) * 16) = make_uint4(0, 0, 0, 0);
                } else if (rows < T) {
                    bad = true;
                }
                uint32_t shi[SCOLS], slo[SCOLS];
                if (!bad && wait_bounded(&sm->s_full[j2], (i >> 1) & 1, abort_flag, budget)) {
                    tc_fence_after_sync();
                    const uint32_t sc = tmem + lane_addr + (j2 * RT + hf) * 2 * RP + hbase;
                    tmem_ld_cols<SCOLS>(sc, shi);
                    tmem_ld_cols<SCOLS>(sc + RP, slo);
                    tmem_wait_ld();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->s_empty[j2]);
                } else {
                    bad = true;
#pragma unroll
                    for (int h = 0; h < SCOLS; ++h) shi[h] = slo[h] = 0u;
                }

                float x[NHW];
                bool need = false;
                {
                    const bool valid = trow < rows;
                    const int over = sg.first + sg.tile(jj) * T + trow - (sg.n - p.Q + 1);
                    const int min_col = over >= 0 ? (over + 1) * p.rb : 0;
#pragma unroll
                    for (int h = 0; h < NHW; ++h) {
                        x[h] = (valid && hbase + h >= min_col)
                                   ? (__uint_as_float(shi[h]) + 0.0625f * __uint_as_float(slo[h])) * f[h]
                                   : -INFINITY;
                        need |= x[h] > m_run[h] + kLazyLog2_8;
                    }
                }
                if (named_bar_any(bar_id, NBAR, bad || need)) {
                    {
                        float wm[NHW];
#pragma unroll
                        for (int h = 0; h < NHW; ++h) wm[h] = x[h];
                        warp_max_transpose8<NHW, C::LOG2NHW>(wm, lane);
                        if (lane < NHW)
                            reinterpret_cast<float *>(&sm->wmax[wg][j2][wq][0])[transpose_head8<NHW, C::LOG2NHW>(lane)] = wm[0];
                    }
                    if (named_bar_any(bar_id, NBAR, bad)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int h4 = 0; h4 < C::NHW4; ++h4) {
                        float4 a = sm->wmax[wg][j2][0][h4];
#pragma unroll
                        for (int q = 1; q < 4 * RS; ++q) {
                            const float4 b = sm->wmax[wg][j2][q][h4];
                            a.x = fmaxf(a.x, b.x);
                            a.y = fmaxf(a.y, b.y);
                            a.z = fmaxf(a.z, b.z);
                            a.w = fmaxf(a.w, b.w);
                        }
                        const float t4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            const int h = h4 * 4 + e4;
                            if (h < NHW) {
                                const float m_new = fmaxf(m_run[h], t4[e4]);
                                alpha[h] = m_new == -INFINITY ? 0.f : ex2_approx(m_run[h] - m_new);
                                m_run[h] = m_new;
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < NHW; ++h) alpha[h] = 1.f;
                }

                // P of this thread's row, as three e4m3 terms, one 16-byte chunk per term (the
                // group's 16 heads; zero bytes for padding heads).
                {
                    float pv[16];
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        if (h < NHW) {
                            pv[h] = x[h] == -INFINITY ? 0.f : ex2_approx(x[h] - m_run[h]);
                            l[h] = l[h] * alpha[h] + pv[h];
                        } else {
                            pv[h] = 0.f;
                        }
                    }
                    uint32_t tw[3][4];
#pragma unroll
                    for (int k = 0; k < 16; k += 4) {
                        if (k < NHW) {
                            uint16_t a0, a1, a2, b0, b1, b2;
                            split3(pv[k], pv[k + 1], a0, a1, a2);
                            split3(pv[k + 2], pv[k + 3], b0, b1, b2);
                            tw[0][k / 4] = static_cast<uint32_t>(a0) | (static_cast<uint32_t>(b0) << 16);
                            tw[1][k / 4] = static_cast<uint32_t>(a1) | (static_cast<uint32_t>(b1) << 16);
                            tw[2][k / 4] = static_cast<uint32_t>(a2) | (static_cast<uint32_t>(b2) << 16);
                        } else {
                            tw[0][k / 4] = tw[1][k / 4] = tw[2][k / 4] = 0u;
                        }
                    }
                    uint8_t *pt = p_base + j2 * C::P_BYTES + p_chunk<RP>(trow, hbase >> 4);
#pragma unroll
                    for (int term = 0; term < 3; ++term)
                        *reinterpret_cast<uint4 *>(pt + term * C::P_TERM) = make_uint4(tw[term][0], tw[term][1], tw[term][2], tw[term][3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->p_full[j2]);

                // O(i-1) was computed against the previous maximum; fold it in and move the
                // sum to the current one.
                if (folds && jj > 0 && !fold_o(i - 1, alpha)) bad = true;
            }
            if (!ok) break;
            if (folds && (bad || !fold_o(i - 1, nullptr))) bad = true;
#pragma unroll
            for (int h = 0; h < NHW; ++h) {
                const float sum = warp_sum_f32(l[h]);
                if (lane == 0) sm->lsum[wg][wq][h] = sum;
            }
            if (named_bar_any(bar_id, NBAR, bad)) {
                ok = false;
                break;
            }
            if (folds && dcol >= 0) {
                float Lh[NHW];
#pragma unroll
                for (int h = 0; h < NHW; ++h) {
                    float L = 0.f;
#pragma unroll
                    for (int q = 0; q < 4 * RS; ++q) L += sm->lsum[wg][q][h];
                    Lh[h] = L;
                }
                if (sg.whole) {
#pragma unroll
                    for (int h = 0; h < NHW; ++h) {
                        const long long orow = out_row(p, sg.b, sg.kvh, sg.hb, hbase + h);
                        if (orow >= 0) p.out[orow * D + dcol] = O[h] * vs / Lh[h];
                    }
                } else {
                    float *slot = p.ws + p.slot_base +
                                  (static_cast<long long>(blockIdx.x) + sg.unit) * p.slot_floats;
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        if (hbase + h < p.RB) slot[(hbase + h) * D + dcol] = O[h] * vs;
                    if (dcol < NHW && hbase + dcol < p.RB) {
                        float m_final = -INFINITY, l_final = 0.f;
#pragma unroll
                        for (int hh = 0; hh < NHW; ++hh)
                            if (hh == dcol) {
                                m_final = m_run[hh];
                                l_final = Lh[hh];
                            }
                        slot[p.RB * D + hbase + dcol] = m_final;
                        slot[p.RB * D + p.RB + hbase + dcol] = l_final;
                    }
                }
            }
            // the next unit rewrites lsum only after every thread has read it, and the slot is
            // complete before the ticket warp is told
            named_bar_sync(bar_id, NBAR);
            if (!sg.whole) {
                if (sm_tid == 0 && npart < 2) mbar_arrive(&sm->pc_full[wg][npart]);
                if (npart < 2) parts[npart] = PendingPiece{sg.uoff, sg.unit, sg.b, sg.kvh, sg.hb, sg.nt};
                ++npart;
            }
            // merge what an earlier piece completed, if its ticket is back
            merge_in(false);
        }
        if (ok && !merge_in(true)) ok = false;
        if (!ok) fail();
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int NH, bool PAGED>
int launch_split_tc8_impl(const TmaMaps &maps, const void *q, const DecodeParams &p,
                          cudaStream_t stream) {
    using C = Tc8Cfg<D, NH>;
    auto kern = split_tc8_kernel<D, NH, PAGED>;
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
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps.k, maps.k8, maps.v, maps.v8,
                           static_cast<const __nv_bfloat16 *>(q), p) != cudaSuccess)
        return GQA_ERR_CUDA;
    return GQA_OK;
}

template <int D, bool PAGED>
int launch_split_tc8_d(const TmaMaps &maps, const void *q, const DecodeParams &p, int nh,
                       cudaStream_t stream) {
    switch (nh) {
        case 1: return launch_split_tc8_impl<D, 1, PAGED>(maps, q, p, stream);
        case 2: return launch_split_tc8_impl<D, 2, PAGED>(maps, q, p, stream);
        case 4: return launch_split_tc8_impl<D, 4, PAGED>(maps, q, p, stream);
        case 8: return launch_split_tc8_impl<D, 8, PAGED>(maps, q, p, stream);
        case 16: return launch_split_tc8_impl<D, 16, PAGED>(maps, q, p, stream);
        default: return launch_split_tc8_impl<D, 32, PAGED>(maps, q, p, stream);  // units have <= 32 columns
    }
}

int heads_bucket8(int heads_per_unit) {
    int nh = 1;
    while (nh < heads_per_unit) nh <<= 1;
    return nh;
}

}  // namespace

// Rows of one tile of the FP8 kernel for a unit of `heads_per_unit` columns.
int tc8_tile_rows(int heads_per_unit) { return heads_bucket8(heads_per_unit) <= 16 ? 256 : 128; }

int launch_split_tc8(const TmaMaps &maps, const void *q, const DecodeParams &p, cudaStream_t stream) {
    const int nh = heads_bucket8(p.RB);
    const bool paged = p.block_table != nullptr;
    if (p.d == 128)
        return paged ? launch_split_tc8_d<128, true>(maps, q, p, nh, stream)
                     : launch_split_tc8_d<128, false>(maps, q, p, nh, stream);
    return paged ? launch_split_tc8_d<64, true>(maps, q, p, nh, stream)
                 : launch_split_tc8_d<64, false>(maps, q, p, nh, stream);
}

}  // namespace gqa
