// Split-KV GQA decode for bf16 caches on sm_100a tensor cores (tcgen05 + TMA).
//
// One persistent CTA per SM walks its range of (unit, tile) work (schedule.cuh).  A tile is
// T = 128 cached rows of one key/value head.  Each K/V tile is read from HBM once, by TMA,
// into a shared-memory ring, and serves every query head of the group ("GQA 阅读笔记",
// Algorithm 2 notes: a good kernel fuses the H/G queries of a group so each cached K vector is
// read once for all of them).  Per tile:
//
//   S^T[128 rows x RP heads] = K_tile[128 x d] . Q^T            (UMMA, M=128, N=RP, K=d)
//   softmax over the 128 rows, online across tiles, in fp32      (4 warps, one row per thread)
//   O^T[d x RP] = V_tile^T[d x 128] . P^T[128 x RP]              (UMMA, M=d, N=RP, K=128)
//
// and the O^T tiles are accumulated with the online-softmax rescale in registers (thread =
// one of the d output columns).  P enters the second product as two bf16 parts (high, and the
// rounding residual) that accumulate into the same TMEM tile, so it carries ~16 significant
// bits rather than 8.  RP is the group's head count padded to 16/32/64; padded heads are
// computed and ignored.  Roles (192 threads):
//   warp 0       TMA producer (q of each unit, K/V tiles); also owns the tensor memory
//   warp 1       UMMA issuer (one elected thread)
//   warps 2..5   softmax / accumulation / epilogue (128 threads)
// Every wait is bounded; on a timeout the CTA drains its in-flight copies and UMMAs, frees
// its tensor memory, sets GQA_STATUS_WAIT_TIMEOUT and returns.
#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {

constexpr unsigned long long kDrainNs = 1000000000ull;  // bound for draining in-flight work

template <int D, int RP>
struct TcCfg {
    static constexpr int T = 128;
    static constexpr int KB = D / 64;                 // 128-byte column blocks of a row
    static constexpr int TILE_BYTES = T * D * 2;      // one K or V tile
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int Q_BYTES = RP * D * 2;
    static constexpr int P_HALF = RP * T * 2;         // P^T in bf16: high part, then low part
    static constexpr int P_BYTES = 2 * P_HALF;
    static constexpr int TMEM_COLS = 4 * RP;          // S^T x2, O^T x2
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, RP, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(D, RP, true, false);

    struct Small {
        uint64_t kv_full[8], kv_empty[8];
        uint64_t q_full[2], q_empty[2];
        uint64_t s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2];
        uint64_t mma_done;
        uint32_t tmem_base;
        int abort;
        int b0;
        int pad_;
        long long begin, end, off0;
        float wmax[2][4][RP];
        float mcur[2][RP];
        float alpha[2][RP];
        float lsum[4][RP];
    };

    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int BASE = 2 * P_BYTES + static_cast<int>(sizeof(Small));
    // two q buffers (the next unit's q loads during the current unit) when two stages still fit
    static constexpr int QB = (SMEM_LIMIT - BASE - 2 * Q_BYTES >= 2 * STAGE_BYTES) ? 2 : 1;
    static constexpr int FIXED = BASE + QB * Q_BYTES;
    static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE_BYTES;
    static constexpr int S = S_FIT > 6 ? 6 : S_FIT;
    static constexpr int SMEM_BYTES = S * STAGE_BYTES + FIXED;
    static_assert(S >= 2, "shared memory too small for a double-buffered ring");
    static_assert(Q_BYTES % 1024 == 0 && P_HALF % 1024 == 0 && STAGE_BYTES % 1024 == 0, "");
};

template <int D, int RP>
__global__ void __launch_bounds__(192, 1)
split_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_k8, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_v8, const DecodeParams p) {
    using C = TcCfg<D, RP>;
    constexpr int T = C::T;
    constexpr int S = C::S;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *const st_base = smem;
    uint8_t *const q_base = smem + S * C::STAGE_BYTES;
    uint8_t *const p_base = q_base + C::QB * C::Q_BYTES;
    auto *const sm = reinterpret_cast<typename C::Small *>(p_base + 2 * C::P_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0 && p.status != nullptr) atomicOr(p.status, GQA_STATUS_INTERNAL);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&sm->kv_full[s], 1);
            mbar_init(&sm->kv_empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm->q_full[j], 1);
            mbar_init(&sm->q_empty[j], 1);
            mbar_init(&sm->s_full[j], 1);
            mbar_init(&sm->s_empty[j], 4);
            mbar_init(&sm->p_full[j], 4);
            mbar_init(&sm->o_full[j], 1);
            mbar_init(&sm->o_empty[j], 4);
        }
        mbar_init(&sm->mma_done, 1);
        sm->abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 1 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_k8);
        prefetch_tmap(&tm_v8);
    }
    // Everything below reads what the previous kernel on the stream (the append) wrote.
    grid_dependency_wait();
    if (warp == 2) {
        long long *hdr = blockIdx.x == 0 ? reinterpret_cast<long long *>(p.ws) : nullptr;
        const CtaRange cr = locate_cta_range(p, blockIdx.x, lane, hdr, blockIdx.x == 0);
        if (lane == 0) {
            sm->begin = cr.begin;
            sm->end = cr.end;
            sm->b0 = cr.b0;
            sm->off0 = cr.off0;
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
    cr.total = 0;
    volatile int *abort_flag = &sm->abort;
    const uint64_t budget = p.wait_ns;

    auto fail = [&]() {
        *abort_flag = 1;
        if (p.status != nullptr) atomicOr(p.status, GQA_STATUS_WAIT_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            SegmentWalker w;
            w.init(p, cr);
            Segment sg;
            int i = 0, sidx = 0;
            bool ok = true;
            while (ok && w.next(sg)) {
                const int qb = sidx % C::QB;
                if (sidx >= C::QB && !wait_bounded(&sm->q_empty[qb], ((sidx / C::QB) - 1) & 1, abort_flag, budget)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&sm->q_full[qb], C::Q_BYTES);
                const int qrow = sg.b * p.H_q + sg.kvh * p.r + sg.hb * p.RB;
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_2d(q_base + qb * C::Q_BYTES + kb * RP * 128, &tm_q, &sm->q_full[qb],
                                kb * 64, qrow);
                ++sidx;
                for (int jj = 0; jj < sg.len; ++jj) {
                    const int st = i % S;
                    if (i >= S && !wait_bounded(&sm->kv_empty[st], ((i / S) - 1) & 1, abort_flag, budget)) {
                        ok = false;
                        break;
                    }
                    const int row0 = (sg.j0 + jj) * T;
                    const int rows = min(T, sg.n - row0);
                    uint8_t *kdst = st_base + st * C::STAGE_BYTES;
                    uint8_t *vdst = kdst + C::TILE_BYTES;
                    if (rows == T) {
                        mbar_arrive_expect_tx(&sm->kv_full[st], C::STAGE_BYTES);
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb) {
                            tma_load_4d(kdst + kb * T * 128, &tm_k, &sm->kv_full[st], kb * 64, sg.kvh, row0, sg.b, pol);
                            tma_load_4d(vdst + kb * T * 128, &tm_v, &sm->kv_full[st], kb * 64, sg.kvh, row0, sg.b, pol);
                        }
                    } else {
                        const int nb = (rows + 7) >> 3;  // 8-row boxes: at most 7 rows past n
                        mbar_arrive_expect_tx(&sm->kv_full[st], 2 * C::KB * nb * 8 * 128);
                        for (int x = 0; x < nb; ++x) {
#pragma unroll
                            for (int kb = 0; kb < C::KB; ++kb) {
                                tma_load_4d(kdst + kb * T * 128 + x * 1024, &tm_k8, &sm->kv_full[st], kb * 64, sg.kvh, row0 + 8 * x, sg.b, pol);
                                tma_load_4d(vdst + kb * T * 128 + x * 1024, &tm_v8, &sm->kv_full[st], kb * 64, sg.kvh, row0 + 8 * x, sg.b, pol);
                            }
                        }
                    }
                    ++i;
                }
            }
            if (!ok) fail();
            // Drain: no copy may still be writing this CTA's shared memory when it exits.
            for (int ii = (i > S ? i - S : 0); ii < i; ++ii)
                wait_bounded(&sm->kv_full[ii % S], (ii / S) & 1, nullptr, kDrainNs);
            for (int ss = (sidx > C::QB ? sidx - C::QB : 0); ss < sidx; ++ss)
                wait_bounded(&sm->q_full[ss % C::QB], (ss / C::QB) & 1, nullptr, kDrainNs);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ UMMA issuer
        if (lane == 0) {
            SegmentWalker w;
            w.init(p, cr);
            Segment sg;
            int i = 0, sidx = 0, pv_next = 0;
            bool ok = true;
            auto issue_pv = [&](int t) -> bool {
                const int j2 = t & 1;
                if (!wait_bounded(&sm->p_full[j2], (t >> 1) & 1, abort_flag, budget)) return false;
                if (t >= 2 && !wait_bounded(&sm->o_empty[j2], ((t >> 1) - 1) & 1, abort_flag, budget)) return false;
                tc_fence_after_sync();
                const uint32_t vaddr = smem_u32(st_base + (t % S) * C::STAGE_BYTES + C::TILE_BYTES);
                const uint32_t paddr = smem_u32(p_base + j2 * C::P_BYTES);
                // O^T = V^T . (P_hi + P_lo)^T: the two bf16 parts of P accumulate into one tile,
                // so P enters the product with ~16 significant bits instead of 8.
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int kk = 0; kk < T / 16; ++kk) {
                        // V^T: M = d (contiguous within 128-byte rows), K = rows; MN-major.
                        const uint64_t a = sdesc_sw128(vaddr + kk * 2048, T * 128, 1024);
                        // P^T: N = heads, K = rows; K-major, 64 rows per 128-byte swizzle row.
                        const uint64_t bdesc = sdesc_sw128(paddr + part * C::P_HALF + (kk >> 2) * RP * 128 + (kk & 3) * 32, 16, 1024);
                        umma_bf16(tmem + 2 * RP + j2 * RP, a, bdesc, C::IDESC_PV, (part | kk) ? 1u : 0u);
                    }
                }
                umma_commit(&sm->o_full[j2]);
                umma_commit(&sm->kv_empty[t % S]);
                return true;
            };
            while (ok && w.next(sg)) {
                const int qb = sidx % C::QB;
                if (!wait_bounded(&sm->q_full[qb], (sidx / C::QB) & 1, abort_flag, budget)) {
                    ok = false;
                    break;
                }
                const uint32_t qaddr = smem_u32(q_base + qb * C::Q_BYTES);
                for (int jj = 0; jj < sg.len; ++jj, ++i) {
                    const int st = i % S;
                    const int j2 = i & 1;
                    if (!wait_bounded(&sm->kv_full[st], (i / S) & 1, abort_flag, budget)) { ok = false; break; }
                    if (i >= 2 && !wait_bounded(&sm->s_empty[j2], ((i >> 1) - 1) & 1, abort_flag, budget)) { ok = false; break; }
                    tc_fence_after_sync();
                    const uint32_t kaddr = smem_u32(st_base + st * C::STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // K tile: M = rows, K = d; K-major.  Q: N = heads, K = d; K-major.
                        const uint64_t a = sdesc_sw128(kaddr + (kk >> 2) * T * 128 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bdesc = sdesc_sw128(qaddr + (kk >> 2) * RP * 128 + (kk & 3) * 32, 16, 1024);
                        umma_bf16(tmem + j2 * RP, a, bdesc, C::IDESC_QK, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&sm->s_full[j2]);
                    const bool last = (jj == sg.len - 1);
                    if (last) umma_commit(&sm->q_empty[qb]);
                    if (pv_next < i) {
                        if (!issue_pv(pv_next)) { ok = false; break; }
                        ++pv_next;
                    }
                    if (last) {
                        if (!issue_pv(i)) { ok = false; break; }
                        pv_next = i + 1;
                    }
                }
                ++sidx;
            }
            if (!ok) fail();
            umma_commit(&sm->mma_done);
            wait_bounded(&sm->mma_done, 0, nullptr, kDrainNs);
        }
    } else {
        // ------------------------------------------------------------------ softmax warps
        const int q4 = warp & 3;               // TMEM lane quadrant this warp may access
        const int row = q4 * 32 + lane;        // tile row of S^T this thread owns
        const int wg_tid = threadIdx.x - 64;   // 0..127
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        // Output column (of d) this thread accumulates: O^T row in TMEM.
        const int dcol = (D == 128) ? row : (lane < 16 ? q4 * 16 + lane : -1);
        SegmentWalker w;
        w.init(p, cr);
        Segment sg;
        int i = 0;
        bool ok = true;
        float O[RP];
        float l[RP];
        while (ok && w.next(sg)) {
            const int nh = min(p.RB, p.r - sg.hb * p.RB);
#pragma unroll
            for (int h = 0; h < RP; ++h) {
                O[h] = 0.f;
                l[h] = 0.f;
            }
            int j2 = 0;
            for (int jj = 0; jj < sg.len; ++jj, ++i) {
                j2 = i & 1;
                const int rows = min(T, sg.n - (sg.j0 + jj) * T);
                if (rows < T) {
                    // Rows past n: zero V in shared memory so that 0-weight rows add exactly 0
                    // (stale or unread data there may hold NaN or Inf).
                    if (!wait_bounded(&sm->kv_full[i % S], (i / S) & 1, abort_flag, budget)) { ok = false; break; }
                    uint8_t *vbase = st_base + (i % S) * C::STAGE_BYTES + C::TILE_BYTES;
                    const int nchunks = (T - rows) * 8;  // 16-byte chunks per column block
                    for (int c = wg_tid; c < nchunks * C::KB; c += 128) {
                        const int kb = c / nchunks;
                        const int rem = c - kb * nchunks;
                        const int rr = rows + (rem >> 3);
                        *reinterpret_cast<uint4 *>(vbase + kb * T * 128 + rr * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                if (!wait_bounded(&sm->s_full[j2], (i >> 1) & 1, abort_flag, budget)) { ok = false; break; }
                tc_fence_after_sync();
                uint32_t sr[RP];
                tmem_ld_cols<RP>(tmem + lane_addr + j2 * RP, sr);
                tmem_wait_ld();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->s_empty[j2]);

                const bool valid = row < rows;
                float x[RP];
#pragma unroll
                for (int h = 0; h < RP; ++h)
                    x[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
#pragma unroll
                for (int h = 0; h < RP; ++h) {
                    if (h < nh) {
                        const float wm = warp_max_f32(x[h]);
                        if (lane == 0) sm->wmax[j2][q4][h] = wm;
                    }
                }
                named_bar_sync(1, 128);
                if (wg_tid < nh) {
                    const int h = wg_tid;
                    const float tmax = fmaxf(fmaxf(sm->wmax[j2][0][h], sm->wmax[j2][1][h]),
                                             fmaxf(sm->wmax[j2][2][h], sm->wmax[j2][3][h]));
                    const float m_old = jj == 0 ? -INFINITY : sm->mcur[j2 ^ 1][h];
                    const float m_new = fmaxf(m_old, tmax);
                    sm->mcur[j2][h] = m_new;
                    sm->alpha[j2][h] = jj == 0 ? 0.f : ex2_approx(m_old - m_new);
                }
                named_bar_sync(1, 128);

                // P^T as bf16 high and low parts (P = hi + lo to ~16 bits), K-major with
                // 128-byte swizzle: head h is row h, tile row r is column r (64 columns per
                // 128-byte row, two column blocks).
                uint8_t *pb = p_base + j2 * C::P_BYTES + (row >> 6) * RP * 128;
                const int col = row & 63;
                const int chunk = col >> 3;
                const int within = (col & 7) * 2;
#pragma unroll
                for (int h = 0; h < RP; ++h) {
                    if (h < nh) {
                        const float pr = ex2_approx(x[h] - sm->mcur[j2][h]);
                        const __nv_bfloat16 hi = __float2bfloat16_rn(pr);
                        const __nv_bfloat16 lo = __float2bfloat16_rn(pr - __bfloat162float(hi));
                        l[h] = l[h] * sm->alpha[j2][h] + pr;
                        uint8_t *dst = pb + h * 128 + ((chunk ^ (h & 7)) << 4) + within;
                        *reinterpret_cast<__nv_bfloat16 *>(dst) = hi;
                        *reinterpret_cast<__nv_bfloat16 *>(dst + C::P_HALF) = lo;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->p_full[j2]);

                if (jj > 0) {
                    // O(i-1) was computed against the previous max; fold it in and move the
                    // running sum to the current max.
                    const int t = i - 1, jt = t & 1;
                    if (!wait_bounded(&sm->o_full[jt], (t >> 1) & 1, abort_flag, budget)) { ok = false; break; }
                    tc_fence_after_sync();
                    uint32_t orr[RP];
                    tmem_ld_cols<RP>(tmem + lane_addr + 2 * RP + jt * RP, orr);
                    tmem_wait_ld();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->o_empty[jt]);
#pragma unroll
                    for (int h = 0; h < RP; ++h)
                        if (h < nh) O[h] = (O[h] + __uint_as_float(orr[h])) * sm->alpha[j2][h];
                }
            }
            if (!ok) break;
            {
                // Last tile of the piece: its O is already relative to the final max.
                const int t = i - 1, jt = t & 1;
                if (!wait_bounded(&sm->o_full[jt], (t >> 1) & 1, abort_flag, budget)) { ok = false; break; }
                tc_fence_after_sync();
                uint32_t orr[RP];
                tmem_ld_cols<RP>(tmem + lane_addr + 2 * RP + jt * RP, orr);
                tmem_wait_ld();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->o_empty[jt]);
#pragma unroll
                for (int h = 0; h < RP; ++h)
                    if (h < nh) O[h] += __uint_as_float(orr[h]);
            }
            // Sum of the softmax numerators over the 128 rows of every tile of the piece.
#pragma unroll
            for (int h = 0; h < RP; ++h) {
                if (h < nh) {
                    const float s = warp_sum_f32(l[h]);
                    if (lane == 0) sm->lsum[q4][h] = s;
                }
            }
            named_bar_sync(1, 128);
            if (dcol >= 0) {
                const int h0 = sg.kvh * p.r + sg.hb * p.RB;
                if (sg.whole) {
                    float *o = p.out + (static_cast<long long>(sg.b) * p.H_q + h0) * D + dcol;
#pragma unroll
                    for (int h = 0; h < RP; ++h) {
                        if (h < nh) {
                            const float L = sm->lsum[0][h] + sm->lsum[1][h] + sm->lsum[2][h] + sm->lsum[3][h];
                            o[static_cast<long long>(h) * D] = O[h] / L;
                        }
                    }
                } else {
                    float *slot = p.ws + p.hdr_floats +
                                  (static_cast<long long>(blockIdx.x) + sg.unit) * p.slot_floats;
#pragma unroll
                    for (int h = 0; h < RP; ++h)
                        if (h < nh) slot[h * D + dcol] = O[h];
                    if (dcol < nh) {
                        const int h = dcol;
                        slot[nh * D + h] = sm->mcur[j2][h];
                        slot[nh * D + nh + h] = sm->lsum[0][h] + sm->lsum[1][h] + sm->lsum[2][h] + sm->lsum[3][h];
                    }
                }
            }
        }
        if (!ok) fail();
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int RP>
static int launch_split_tc_impl(const TmaMaps &maps, const DecodeParams &p, cudaStream_t stream) {
    using C = TcCfg<D, RP>;
    auto kern = split_tc_kernel<D, RP>;
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
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps.q, maps.k, maps.k8, maps.v, maps.v8, p) != cudaSuccess)
        return GQA_ERR_CUDA;
    return GQA_OK;
}

int launch_split_tc(const TmaMaps &maps, const DecodeParams &p, int rp, cudaStream_t stream) {
    if (p.d == 128) {
        if (rp == 16) return launch_split_tc_impl<128, 16>(maps, p, stream);
        if (rp == 32) return launch_split_tc_impl<128, 32>(maps, p, stream);
        return launch_split_tc_impl<128, 64>(maps, p, stream);
    }
    if (rp == 16) return launch_split_tc_impl<64, 16>(maps, p, stream);
    if (rp == 32) return launch_split_tc_impl<64, 32>(maps, p, stream);
    return launch_split_tc_impl<64, 64>(maps, p, stream);
}

}  // namespace gqa
