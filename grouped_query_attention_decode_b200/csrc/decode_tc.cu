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
//   O^T[d x PN] = V_tile^T[d x 128] . [P_hi | P_lo]^T            (UMMA, M=d, N=PN, K=128)
//
// (tiles of 256 rows at d = 64 for units of up to 8 columns: two S MMAs, two rows per thread,
// K = 256 for the second product; PN = 2*RP, or 16 for units of up to 8 columns)
//
// and the O^T tiles are accumulated with the online-softmax rescale in registers (thread =
// one of the d output columns).  P enters the second product as two bf16 parts (high, and the
// rounding residual) side by side, summed when the tile is read back, so it carries ~16
// significant bits rather than 8.  NH is the group's head count rounded up to a power of two
// (1..64) and RP = max(16, NH) the UMMA N; padded heads are computed and ignored.
// Roles (64 + 128 * NWG + 32 threads):
//   warp 0       TMA producer (q of each unit, K/V tiles); also owns the tensor memory
//   warp 1       UMMA issuer (one elected thread, event loop)
//   warps 2..    NWG softmax / accumulation / epilogue warpgroups of 128 threads, each owning
//                a slice of the group's query heads (one warpgroup up to 16 heads)
//   last warp    ticket warp: takes the tickets of the pieces cut from units (schedule.cuh);
//                under a fused append it also writes the appended rows into the cache and over
//                the copies of the tiles that hold them
// Every wait is bounded; on a timeout the CTA drains its in-flight copies and UMMAs, frees
// its tensor memory, sets GQA_STATUS_WAIT_TIMEOUT and returns.
#include <cstdint>

#include "device.cuh"
#include "gqa.h"
#include "launch.h"
#include "schedule.cuh"

namespace gqa {

constexpr unsigned long long kDrainNs = 1000000000ull;  // bound for draining in-flight work
// Scores may exceed the running maximum by this much (log2 units) before it is raised.
constexpr float kLazyLog2 = 8.0f;

template <int D, int NH>
struct TcCfg {
    static constexpr int RP = NH < 16 ? 16 : NH;      // UMMA N of S^T = K.Q^T
    // Rows per softmax thread: 64-wide heads of groups up to 8 columns take 256-row tiles (two
    // rows a thread, S^T as two 128-lane halves), so that a stage carries 64 KB as at d = 128
    // and the per-tile chain runs half as often; 128-row tiles otherwise.
    static constexpr int RPT = (D == 64 && NH <= 8) ? 2 : 1;
    static constexpr int T = 128 * RPT;
    static constexpr int KB = D / 64;                 // 128-byte column blocks of a row
    static constexpr int TILE_BYTES = T * D * 2;      // one K or V tile
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int Q_BYTES = RP * D * 2;
    // P^T in bf16, MN-major: tile row r (the K index) holds PN = 2*LO values, the high parts
    // of the heads at [0, LO) and their low parts at [LO, 2*LO).  LO = RP, except for units of
    // up to 8 columns, where one 16-byte chunk holds the 8 high parts and the next the 8 low
    // parts (LO = 8): P is then half the size, so that two P buffers fit beside a three-stage
    // ring of 64 KB stages.  Rows are 32 bytes (32-byte swizzle), 64 bytes (RP = 16, 64-byte
    // swizzle) or 128 bytes (RP >= 32, 128-byte swizzle); PN > 64 values take two 128-byte atoms.
    static constexpr int LO = NH <= 8 ? 8 : RP;
    static constexpr int PN = 2 * LO;                 // UMMA N of O^T = V^T.P^T
    static constexpr int P_ROWB = 2 * PN >= 128 ? 128 : 2 * PN;
    static constexpr int P_ATOMB = T * P_ROWB;
    static constexpr uint32_t P_LAYOUT = P_ROWB == 128 ? 2u : (P_ROWB == 64 ? 4u : 6u);
    static constexpr int P_BYTES = PN * T * 2;
    // TMEM columns: S^T (RPT halves of RP columns) x2 buffers, then O^T (PN: high, low) x2
    static constexpr int S_BUF = RPT * RP;
    static constexpr int O_COL = 2 * S_BUF;
    static constexpr int OB = PN;                     // columns of one O^T buffer
    static constexpr int TMEM_USED = 2 * S_BUF + 2 * OB;
    static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, RP, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(D, PN, true, true);
    // Softmax warpgroups: one for up to 16 heads, else one per 16 heads (heads are
    // independent, so the groups split them and never exchange data).
    static constexpr int NWG = NH >= 32 ? NH / 16 : 1;
    static constexpr int NHW = NH / NWG;              // heads per warpgroup
    static constexpr int TICKET_WARP = 2 + 4 * NWG;
    static constexpr int THREADS = 64 + 128 * NWG + 32;
    static constexpr int NHW4 = (NHW + 3) / 4;
    static constexpr int LOG2NHW = NHW >= 16 ? 4 : NHW >= 8 ? 3 : NHW >= 4 ? 2 : NHW >= 2 ? 1 : 0;

    struct Small {
        // K and V of a stage land on separate barriers: S = K.Q^T starts as soon as K is in,
        // while V is still on its way; the stage is released after P.V
        uint64_t k_full[8], v_full[8], kv_empty[8];
        // fused append: the copies (K, V) of a tile that holds the appended row
        uint64_t apk_full[8], apv_full[8];
        uint64_t q_full[2], q_empty[2];
        uint64_t s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2];
        uint64_t mma_done;
        uint64_t pc_full[kPieceGroups][2];  // a group's partial piece is in its slot
        uint64_t tk_done[kPieceGroups][2];  // its ticket is taken: tk_last says if it was the last
        int tk_last[kPieceGroups][2];  // a group's partial piece is in its slot
        uint32_t tmem_base;
        int abort;
        int b0, bl;
        long long begin, end, off0, offl, total;
        float4 wmax[NWG][2][4][NHW4];  // per group, tile parity, warp: per-head warp maxima
        float lsum[NWG][4][NHW];
    };

    static constexpr int SMEM_LIMIT = 232448;
    // Ring stages that fit next to pb P^T buffers and qb q buffers.
    static constexpr int fit(int pb, int qb) {
        return (SMEM_LIMIT - pb * P_BYTES - static_cast<int>(sizeof(Small)) - qb * Q_BYTES) / STAGE_BYTES;
    }
    // Two P^T buffers let the softmax write tile i's P while the tensor cores still read tile
    // i-1's; one buffer (the softmax then waits for the previous P.V before it writes P) when
    // that is what buys the ring a third stage.  Two q buffers (the next unit's q loads during
    // the current unit) when two stages still fit.
    static constexpr int PB = (fit(2, 2) < 3 && fit(1, 2) >= 3) ? 1 : 2;
    static constexpr int QB = fit(PB, 2) >= 2 ? 2 : 1;
    static constexpr int BASE = PB * P_BYTES + static_cast<int>(sizeof(Small));
    static constexpr int FIXED = BASE + QB * Q_BYTES;
    static constexpr int S_FIT = (SMEM_LIMIT - FIXED) / STAGE_BYTES;
    static constexpr int S = S_FIT > 6 ? 6 : S_FIT;
    static constexpr int SMEM_BYTES = S * STAGE_BYTES + FIXED;
    static_assert(S >= 2, "shared memory too small for a double-buffered ring");
    static_assert(Q_BYTES % 1024 == 0 && P_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "");
};

// Maximum over the warp's 32 lanes of each of v[0..NH): NH-1 shuffles halve the values per lane,
// then 5 - log2(NH) butterflies finish.  Lane l ends with, in v[0], the result for head
// sum_s bit_s(l) * NH / 2^(s+1) (the bit-reversed low bits of l).
template <int NH, int LOG2NH>
__device__ __forceinline__ void warp_max_transpose(float (&v)[NH], int lane) {
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
__device__ __forceinline__ int transpose_head(int lane) {
    int h = 0;
#pragma unroll
    for (int s = 0; s < LOG2NH; ++s) h += ((lane >> s) & 1) * (NH >> (s + 1));
    return h;
}

// Add a byte offset to a shared-memory descriptor's start address (bits 0-13, 16-byte units).
// Shared addresses stay below 2^18, so the field cannot carry into the next one.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) {
    return desc + static_cast<uint64_t>(bytes >> 4);
}

// The ticket warp under a fused append (gqa_kv_append_decode).  Besides the partial pieces'
// tickets (run_ticket_warp), it owns the appended rows: for every tile that holds a unit's row
// n - 1, it writes the new K and V rows (k_new, v_new) to the cache for later steps and, once
// the tile's K copy has landed (it completes on apk_full instead of k_full), writes the K row
// over the row the copy brought into the ring stage and completes the stage's k_full itself,
// which releases the tile to S = K.Q^T as for any other tile; then the same for V (apv_full,
// v_full), so the scores never wait for the V half.  The copy may read the row before or after
// the cache write; nothing else in the kernel reads it.
//
// Both kinds of event come in the CTA's walk order, and every wait blocks (a blocking mbarrier
// wait wakes as soon as its phase completes, where polling both kinds from one loop with a
// back-off takes the tickets late).  A piece that ends its unit computes the
// unit's last tile -- the patched one -- first, so segment s's patch is due while segment s - 1
// is still being computed: the ticket of a partial segment is therefore taken after the next
// segment's patch, which keeps the patch ahead of the scores that wait for it.  No ticket is
// urgent before the CTA's last piece, whose ticket follows no patch.  Returns false when a
// wait ran out.
template <int D, int T, int NG, int S, int STAGE_BYTES, int TILE_BYTES>
__device__ bool append_ticket_warp(const DecodeParams &p, const CtaRange &cr, uint8_t *st_base,
                                   uint64_t *k_full, uint64_t *v_full, uint64_t *apk_full,
                                   uint64_t *apv_full, uint64_t (*pc_full)[2],
                                   uint64_t (*tk_done)[2], int (*tk_last)[2], int lane,
                                   const volatile int *abort_flag, uint64_t budget) {
    constexpr int CH = D / 8;  // 16-byte chunks of a cached row of one head
    const bool mine = lane < 2 * CH;
    const int half = lane / CH, c = lane % CH;
    SegmentWalker w;
    w.init(p, cr);
    Segment sg, pend;
    bool has_pend = false;
    int tile_r = 0;  // walk index of the next segment's first tile
    int k = 0;       // partial pieces seen (a CTA has at most two)
    // Per stage, the parity of its next apk_full / apv_full phase: a stage's patched copies
    // complete in order, and the producer issues the next one only after this warp released the
    // previous (k_full, v_full -> S.K^T, P.V -> kv_empty), so the phases never run ahead of this
    // warp.
    uint32_t ap_phase = 0;
    auto take = [&](const Segment &ps, int kk) {
        for (int g = 0; g < NG; ++g) {
            const bool got = wait_bounded(&pc_full[g][kk], 0, abort_flag, budget);
            if (!__all_sync(kFullMask, got)) return false;
            if (lane == 0) {
                int c0, c1;
                tk_last[g][kk] = take_ticket(p, ps.unit, g) == unit_pieces(ps.uoff, ps.nt, cr.total, p.G, c0, c1) - 1;
                mbar_arrive(&tk_done[g][kk]);
            }
        }
        return true;
    };
    while (w.next(sg)) {
        const int first = tile_r;
        tile_r += sg.len;
        if (sg.appended && sg.j0 + sg.len == sg.nt) {
            // the piece computes the unit's last tile first: walk index `first`
            const int st = first % S;
            const int rrow = (sg.n - 1) - (sg.first + (sg.nt - 1) * T);
            // the new row: one 16-byte chunk of K (lanes < CH) or V (the next CH lanes) per
            // lane, written to the cache at once
            uint4 chunk = make_uint4(0, 0, 0, 0);
            if (mine) {
                const long long src = (static_cast<long long>(sg.b) * p.H_kv + sg.kvh) * CH + c;
                chunk = __ldg(static_cast<const uint4 *>(half ? p.v_new : p.k_new) + src);
                const long long dst = ((static_cast<long long>(sg.b) * p.L_max + (sg.n - 1)) * p.H_kv + sg.kvh) * CH + c;
                static_cast<uint4 *>(half ? p.v_cache : p.k_cache)[dst] = chunk;
            }
            const uint32_t par = (ap_phase >> st) & 1u;
            for (int hv = 0; hv < 2; ++hv) {
                const bool landed = wait_bounded(hv == 0 ? &apk_full[st] : &apv_full[st], par, abort_flag, budget);
                if (!__all_sync(kFullMask, landed)) return false;
                if (mine && half == hv) {
                    // row rrow of the stage's K or V tile: 64-column blocks of T rows of 128
                    // bytes, the 16-byte chunks of a row XOR-swizzled by the row's low three bits
                    uint8_t *base = st_base + st * STAGE_BYTES + hv * TILE_BYTES;
                    const int kb = c >> 3, cc = c & 7;
                    *reinterpret_cast<uint4 *>(base + kb * T * 128 + rrow * 128 + ((cc ^ (rrow & 7)) << 4)) = chunk;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(hv == 0 ? &k_full[st] : &v_full[st]);
            }
            ap_phase ^= 1u << st;
        }
        if (has_pend) {
            if (!take(pend, k - 1)) return false;
            has_pend = false;
        }
        if (!sg.whole && k < 2) {
            pend = sg;
            has_pend = true;
            ++k;
        }
    }
    if (has_pend && !take(pend, k - 1)) return false;
    return true;
}

template <int D, int NH, bool PAGED>
__global__ void __launch_bounds__(TcCfg<D, NH>::THREADS, 1)
split_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_k8, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_v8, const DecodeParams p) {
    using C = TcCfg<D, NH>;
    constexpr int T = C::T;
    constexpr int S = C::S;
    constexpr int RP = C::RP;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *const st_base = smem;
    uint8_t *const q_base = smem + S * C::STAGE_BYTES;
    uint8_t *const p_base = q_base + C::QB * C::Q_BYTES;
    auto *const sm = reinterpret_cast<typename C::Small *>(p_base + C::PB * C::P_BYTES);

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
            mbar_init(&sm->apk_full[s], 1);
            mbar_init(&sm->apv_full[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&sm->q_full[j], 1);
            mbar_init(&sm->q_empty[j], 1);
            mbar_init(&sm->s_full[j], 1);
            mbar_init(&sm->s_empty[j], 4 * C::NWG);
            mbar_init(&sm->p_full[j], 4 * C::NWG);
            mbar_init(&sm->o_full[j], 1);
            mbar_init(&sm->o_empty[j], 4 * C::NWG);
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
    // q rows past a unit's columns are never loaded: zero them once so padded columns see zeros
    for (int c = threadIdx.x; c < C::QB * C::Q_BYTES / 16; c += C::THREADS)
        reinterpret_cast<uint4 *>(q_base)[c] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
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
        // ------------------------------------------------------------------ TMA producer
        // The whole warp walks the tile line; lane 0 waits on the barriers and issues the
        // copies.  In a paged cache each lane instead owns one box of a tile: it loads that
        // box's page id kPageAhead tiles ahead of the copy, so the lookup's latency hides behind
        // the pipeline, and issues the box's copies itself.
        const uint64_t pol = l2_policy_evict_first();
        SegmentWalker w;
        w.init(p, cr);
        Segment sg;
        int i = 0, sidx = 0;
        bool ok = true;
        uint32_t ap_mask = 0, ap_par = 0;  // fused append: stages whose copy lands on apk/apv_full
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
        while (ok && w.next(sg)) {
            const int qb = sidx % C::QB;
            bool got = true;
            if (lane == 0 && sidx >= C::QB)
                got = wait_bounded(&sm->q_empty[qb], ((sidx / C::QB) - 1) & 1, abort_flag, budget);
            if (!__shfl_sync(kFullMask, got, 0)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                // q of the unit: rows (token j, head h') of q viewed as (d, H_q, B*Q)
                mbar_arrive_expect_tx(&sm->q_full[qb], p.q_box_bytes);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(q_base + qb * C::Q_BYTES + kb * RP * 128, &tm_q, &sm->q_full[qb],
                                kb * 64, sg.kvh * p.r + sg.hb * p.rb, sg.b * p.Q);
            }
            ++sidx;
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
                got = true;
                if (lane == 0 && i >= S)
                    got = wait_bounded(&sm->kv_empty[st], ((i / S) - 1) & 1, abort_flag, budget);
                if (!__shfl_sync(kFullMask, got, 0)) {
                    ok = false;
                    break;
                }
                uint8_t *kdst = st_base + st * C::STAGE_BYTES;
                uint8_t *vdst = kdst + C::TILE_BYTES;
                // K lands on k_full, V on v_full.  A tile that holds a fused append's row lands
                // on apk_full and apv_full instead; the ticket warp writes the row over each
                // copy and then completes k_full and v_full itself.
                uint64_t *kfull = &sm->k_full[st], *vfull = &sm->v_full[st];
                ap_mask &= ~(1u << st);
                if (!PAGED && sg.appended && sg.last_tile(jj)) {
                    kfull = &sm->apk_full[st];
                    vfull = &sm->apv_full[st];
                    ap_mask |= 1u << st;   // the copy now in flight in stage st lands on apk/apv_full
                    ap_par ^= 1u << st;    // with the phase parity before this flip
                }
                if constexpr (PAGED) {
                    // boxes of min(page_size, T) rows, or 8 rows for a partial tile
                    const int boxr = rows == T ? min(p.page_size, T) : 8;
                    const int nbox = rows == T ? T / boxr : (rows + 7) >> 3;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&sm->k_full[st], C::KB * nbox * boxr * 128);
                        mbar_arrive_expect_tx(&sm->v_full[st], C::KB * nbox * boxr * 128);
                    }
                    __syncwarp();
                    if (lane < nbox) {
                        if (pg < 0 || pg >= p.n_pages) {
                            if (p.status != nullptr) atomicOr(p.status, GQA_STATUS_PAGE_RANGE);
                            pg = 0;
                        }
                        const CUtensorMap *mk = rows == T ? &tm_k : &tm_k8;
                        const CUtensorMap *mv = rows == T ? &tm_v : &tm_v8;
                        const int pr = (row0 + lane * boxr) % p.page_size;
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb) {
                            tma_load_4d(kdst + kb * T * 128 + lane * boxr * 128, mk, &sm->k_full[st], kb * 64, sg.kvh, pr, pg, pol);
                            tma_load_4d(vdst + kb * T * 128 + lane * boxr * 128, mv, &sm->v_full[st], kb * 64, sg.kvh, pr, pg, pol);
                        }
                    }
                } else if (lane == 0) {
                    if (rows == T) {
                        mbar_arrive_expect_tx(kfull, C::TILE_BYTES);
                        mbar_arrive_expect_tx(vfull, C::TILE_BYTES);
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb)
                            tma_load_4d(kdst + kb * T * 128, &tm_k, kfull, kb * 64, sg.kvh, row0, sg.b, pol);
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb)
                            tma_load_4d(vdst + kb * T * 128, &tm_v, vfull, kb * 64, sg.kvh, row0, sg.b, pol);
                    } else {
                        const int nb = (rows + 7) >> 3;  // 8-row boxes: at most 7 rows past n
                        mbar_arrive_expect_tx(kfull, C::KB * nb * 8 * 128);
                        mbar_arrive_expect_tx(vfull, C::KB * nb * 8 * 128);
                        for (int x = 0; x < nb; ++x) {
#pragma unroll
                            for (int kb = 0; kb < C::KB; ++kb)
                                tma_load_4d(kdst + kb * T * 128 + x * 1024, &tm_k8, kfull, kb * 64, sg.kvh, row0 + 8 * x, sg.b, pol);
                        }
                        for (int x = 0; x < nb; ++x) {
#pragma unroll
                            for (int kb = 0; kb < C::KB; ++kb)
                                tma_load_4d(vdst + kb * T * 128 + x * 1024, &tm_v8, vfull, kb * 64, sg.kvh, row0 + 8 * x, sg.b, pol);
                        }
                    }
                }
                ++i;
            }
        }
        if (lane == 0) {
            if (!ok) fail();
            // Drain: no copy may still be writing this CTA's shared memory when it exits (a
            // patched tile's copies complete on apk_full / apv_full, which the ticket warp waits for).
            for (int ii = (i > S ? i - S : 0); ii < i; ++ii) {
                const int st = ii % S;
                if (ap_mask & (1u << st)) {
                    wait_bounded(&sm->apk_full[st], ((ap_par >> st) & 1u) ^ 1u, nullptr, kDrainNs);
                    wait_bounded(&sm->apv_full[st], ((ap_par >> st) & 1u) ^ 1u, nullptr, kDrainNs);
                } else {
                    wait_bounded(&sm->k_full[st], (ii / S) & 1, nullptr, kDrainNs);
                    wait_bounded(&sm->v_full[st], (ii / S) & 1, nullptr, kDrainNs);
                }
            }
            for (int ss = (sidx > C::QB ? sidx - C::QB : 0); ss < sidx; ++ss)
                wait_bounded(&sm->q_full[ss % C::QB], (ss / C::QB) & 1, nullptr, kDrainNs);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ UMMA issuer
        // An event loop: a tile's S^T = K.Q^T is issued once its K tile has landed and its S
        // buffer is free; its O^T = V^T.P^T once its V tile has landed and the softmax warps
        // have written its P.  Each is issued as soon as it is ready, so releasing a stage
        // never waits for the next tile's data to arrive.
        if (lane == 0) {
            // K tile and Q: K-major (rows / heads by d), 8-row groups 1024 B apart.
            // V^T: MN-major (d by rows): the two 64-column blocks T*128 B apart.
            // P^T: MN-major (PN values per tile row), 8-row groups 8*P_ROWB apart.
            const uint64_t dk0 = sdesc_sw128(smem_u32(st_base), 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_u32(st_base + C::TILE_BYTES), T * 128, 1024);
            const uint64_t dq0 = sdesc_sw128(smem_u32(q_base), 16, 1024);
            const uint64_t dp0 = sdesc_swz(smem_u32(p_base), C::P_ATOMB, 8 * C::P_ROWB, C::P_LAYOUT);
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
                if (qk_more) {
                    const int qb = sidx % C::QB;
                    if (!q_ready) q_ready = mbar_test_wait(&sm->q_full[qb], (sidx / C::QB) & 1);
                    const int st = qk_t % S;
                    const int j2 = qk_t & 1;
                    if (q_ready && mbar_test_wait(&sm->k_full[st], (qk_t / S) & 1) &&
                        (qk_t < 2 || mbar_test_wait(&sm->s_empty[j2], ((qk_t >> 1) - 1) & 1))) {
                        tc_fence_after_sync();
                        const uint64_t dk = desc_add(dk0, st * C::STAGE_BYTES);
                        const uint64_t dq = desc_add(dq0, qb * C::Q_BYTES);
#pragma unroll
                        for (int hf = 0; hf < C::RPT; ++hf) {  // 128-row halves of the tile
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off_k = (kk >> 2) * T * 128 + hf * 128 * 128 + (kk & 3) * 32;
                                const uint32_t off_q = (kk >> 2) * RP * 128 + (kk & 3) * 32;
                                umma_bf16(tmem + j2 * C::S_BUF + hf * RP, desc_add(dk, off_k), desc_add(dq, off_q),
                                          C::IDESC_QK, kk > 0 ? 1u : 0u);
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
                if (pv_t < qk_t) {
                    const int j2 = pv_t & 1;
                    if (mbar_test_wait(&sm->p_full[j2], (pv_t >> 1) & 1) &&
                        mbar_test_wait(&sm->v_full[pv_t % S], (pv_t / S) & 1) &&
                        (pv_t < 2 || mbar_test_wait(&sm->o_empty[j2], ((pv_t >> 1) - 1) & 1))) {
                        tc_fence_after_sync();
                        const uint64_t dv = desc_add(dv0, (pv_t % S) * C::STAGE_BYTES);
                        const uint64_t dp = desc_add(dp0, (j2 % C::PB) * C::P_BYTES);
                        // O^T[:, 0:RP] = V^T.P_hi^T and O^T[:, RP:2RP] = V^T.P_lo^T in one
                        // N = 2*RP product.
#pragma unroll
                        for (int kk = 0; kk < T / 16; ++kk) {
                            umma_bf16(tmem + C::O_COL + j2 * C::OB, desc_add(dv, kk * 2048),
                                      desc_add(dp, kk * 16 * C::P_ROWB), C::IDESC_PV, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&sm->o_full[j2]);
                        umma_commit(&sm->kv_empty[pv_t % S]);
                        ++pv_t;
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
            wait_bounded(&sm->mma_done, 0, nullptr, kDrainNs);
        }
    } else if (warp == C::TICKET_WARP) {
        // ------------------------------------------------------------------ ticket warp
        if (!PAGED && p.append) {
            if (!append_ticket_warp<D, T, C::NWG, S, C::STAGE_BYTES, C::TILE_BYTES>(
                    p, cr, st_base, sm->k_full, sm->v_full, sm->apk_full, sm->apv_full, sm->pc_full, sm->tk_done,
                    sm->tk_last, lane, abort_flag, budget) &&
                lane == 0)
                fail();
        } else {
            run_ticket_warp<C::NWG>(p, cr, sm->pc_full, sm->tk_done, sm->tk_last, lane, abort_flag, budget);
        }
    } else {
        // ------------------------------------------------------------------ softmax warps
        // NWG warpgroups of four warps; warpgroup g owns query heads [g*NHW, (g+1)*NHW) of the
        // unit.  Heads are independent, so the groups never exchange data: each has its own
        // named barrier (1 + g) and its own per-head state.
        constexpr int NHW = C::NHW;
        constexpr int SCOLS = C::NWG == 1 ? RP : NHW;  // S^T columns this group loads
        const int wg = (warp - 2) >> 2;
        const int hbase = wg * NHW;
        const uint32_t bar_id = 1 + wg;
        const int q4 = warp & 3;                 // TMEM lane quadrant this warp may access
        const int row = q4 * 32 + lane;          // tile row of S^T this thread owns
        const int sm_tid = threadIdx.x - 64;     // 0 .. 128*NWG-1
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        // Output column (of d) this thread accumulates: O^T row in TMEM.
        const int dcol = (D == 128) ? row : (lane < 16 ? q4 * 16 + lane : -1);
        SegmentWalker w;
        w.init(p, cr);
        Segment sg;
        int i = 0;
        bool ok = true;
        float O[NHW], l[NHW], m_run[NHW], alpha[NHW];
        int npart = 0, nmerged = 0;  // partial pieces handed to the ticket warp, reports taken
        PendingPiece parts[2];
        auto merge_in = [&](bool block) {
            return merge_reported(p, cr.total, wg, hbase, hbase + NHW, sm_tid - 128 * wg, 128, sm->tk_done[wg], sm->tk_last[wg],
                                  parts, npart, nmerged, block, abort_flag, budget,
                                  [&](bool pred) { return named_bar_any(bar_id, 128, pred); });
        };
        // units with no rows get zeros (while the first tiles are still on their way)
        zero_empty_units(p, blockIdx.x, sm_tid, 128 * C::NWG);
        while (ok && w.next(sg)) {
#pragma unroll
            for (int h = 0; h < NHW; ++h) {
                O[h] = 0.f;
                l[h] = 0.f;
                m_run[h] = -INFINITY;
            }
            // A failed wait sets `bad`; the threads then agree at the next named barrier
            // (named_bar_any) and leave together, so no warp is left waiting at a barrier.
            bool bad = false;
            for (int jj = 0; jj < sg.len; ++jj, ++i) {
                const int j2 = i & 1;
                const int rows = min(T, sg.n - sg.first - sg.tile(jj) * T);
                if (rows < T && !bad && wait_bounded(&sm->v_full[i % S], (i / S) & 1, abort_flag, budget)) {
                    // Rows past n: zero V in shared memory so that 0-weight rows add exactly 0
                    // (stale or unread data there may hold NaN or Inf).
                    uint8_t *vbase = st_base + (i % S) * C::STAGE_BYTES + C::TILE_BYTES;
                    const int nchunks = (T - rows) * 8;  // 16-byte chunks per column block
                    for (int c = sm_tid; c < nchunks * C::KB; c += 128 * C::NWG) {
                        const int kb = c / nchunks;
                        const int rem = c - kb * nchunks;
                        const int rr = rows + (rem >> 3);
                        *reinterpret_cast<uint4 *>(vbase + kb * T * 128 + rr * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
                    }
                } else if (rows < T) {
                    bad = true;
                }
                uint32_t sr[C::RPT][SCOLS];
                if (!bad && wait_bounded(&sm->s_full[j2], (i >> 1) & 1, abort_flag, budget)) {
                    tc_fence_after_sync();
#pragma unroll
                    for (int hf = 0; hf < C::RPT; ++hf)
                        tmem_ld_cols<SCOLS>(tmem + lane_addr + j2 * C::S_BUF + hf * RP + hbase, sr[hf]);
                    tmem_wait_ld();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->s_empty[j2]);
                } else {
                    bad = true;
#pragma unroll
                    for (int hf = 0; hf < C::RPT; ++hf)
#pragma unroll
                        for (int h = 0; h < SCOLS; ++h) sr[hf][h] = 0u;
                }

                // This thread's rows of the tile: row, and row + 128 with 256-row tiles.
                float x[C::RPT][NHW];
#pragma unroll
                for (int hf = 0; hf < C::RPT; ++hf) {
                    const int trow = row + 128 * hf;
                    const bool valid = trow < rows;
                    // Several query tokens: column j * rb + h' sees rows < n - Q + 1 + j, so a row
                    // `over` rows past n - Q is visible only to columns >= (over + 1) * rb.
                    const int over = sg.first + sg.tile(jj) * T + trow - (sg.n - p.Q + 1);
                    const int min_col = over >= 0 ? (over + 1) * p.rb : 0;
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        x[hf][h] = (valid && hbase + h >= min_col) ? __uint_as_float(sr[hf][h]) * p.scale_log2 : -INFINITY;
                }
                // Lazy rescaling.  The running maximum m_run only has to keep the exponents in
                // range, so it is raised -- through an exchange of the warps' tile maxima -- only
                // when some score of the tile exceeds it by more than kLazyLog2; otherwise every
                // p = 2^(x - m_run) <= 2^kLazyLog2 and nothing is rescaled.  The result is exact
                // either way: P, the running sums and O always share one reference.
                bool need = false;
#pragma unroll
                for (int hf = 0; hf < C::RPT; ++hf)
#pragma unroll
                    for (int h = 0; h < NHW; ++h) need |= x[hf][h] > m_run[h] + kLazyLog2;
                if (named_bar_any(bar_id, 128, bad || need)) {
                    // Per-head maximum over the warp's rows, then over the four warps.
                    {
                        float wm[NHW];
#pragma unroll
                        for (int h = 0; h < NHW; ++h) {
                            wm[h] = x[0][h];
#pragma unroll
                            for (int hf = 1; hf < C::RPT; ++hf) wm[h] = fmaxf(wm[h], x[hf][h]);
                        }
                        warp_max_transpose<NHW, C::LOG2NHW>(wm, lane);
                        if (lane < NHW)
                            reinterpret_cast<float *>(&sm->wmax[wg][j2][q4][0])[transpose_head<NHW, C::LOG2NHW>(lane)] = wm[0];
                    }
                    if (named_bar_any(bar_id, 128, bad)) {
                        ok = false;
                        break;
                    }
                    // Every thread forms the tile maximum of each of its heads from the four
                    // warp maxima; the running maximum stays identical in all threads.
#pragma unroll
                    for (int h4 = 0; h4 < C::NHW4; ++h4) {
                        const float4 a = sm->wmax[wg][j2][0][h4], b = sm->wmax[wg][j2][1][h4];
                        const float4 c = sm->wmax[wg][j2][2][h4], e = sm->wmax[wg][j2][3][h4];
                        const float t4[4] = {fmaxf(fmaxf(a.x, b.x), fmaxf(c.x, e.x)),
                                             fmaxf(fmaxf(a.y, b.y), fmaxf(c.y, e.y)),
                                             fmaxf(fmaxf(a.z, b.z), fmaxf(c.z, e.z)),
                                             fmaxf(fmaxf(a.w, b.w), fmaxf(c.w, e.w))};
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

                // P = hi + lo in bf16 (~16 significant bits).  This thread's tile rows are K rows
                // of the MN-major P^T: high parts at values [0, RP), low parts at [RP, 2RP),
                // written as 16-byte chunks of 8 heads.
                {
                    constexpr int HALF_VALS = C::P_ROWB / 2;  // bf16 values per atom row
#pragma unroll
                    for (int h = 0; h < NHW; ++h) {
                        // x now holds p; a column with no visible row yet (several query tokens)
                        // keeps p = 0 rather than exp(-inf + inf)
#pragma unroll
                        for (int hf = 0; hf < C::RPT; ++hf)
                            x[hf][h] = x[hf][h] == -INFINITY ? 0.f : ex2_approx(x[hf][h] - m_run[h]);
                        l[h] = l[h] * alpha[h] + x[0][h];
#pragma unroll
                        for (int hf = 1; hf < C::RPT; ++hf) l[h] += x[hf][h];
                    }
                    // One P^T buffer: the previous tile's P.V must have read it (its O is folded
                    // below, after this tile's P is handed over).
                    if (C::PB == 1 && jj > 0 && !bad &&
                        !wait_bounded(&sm->o_full[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, budget))
                        bad = true;
#pragma unroll
                    for (int hf = 0; hf < C::RPT; ++hf) {
                    const int trow = row + 128 * hf;
                    uint8_t *prow = p_base + (j2 % C::PB) * C::P_BYTES + trow * C::P_ROWB;
                    const int swz = C::P_ROWB == 128 ? (trow & 7) : (C::P_ROWB == 64 ? ((trow >> 1) & 3) : ((trow >> 2) & 1));
#pragma unroll
                    for (int c8 = 0; c8 < (NHW + 7) / 8; ++c8) {
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int w2 = 0; w2 < 4; ++w2) {
                            const int h = c8 * 8 + 2 * w2;
                            const float a = h < NHW ? x[hf][h] : 0.f;
                            const float b = h + 1 < NHW ? x[hf][h + 1] : 0.f;
                            const __nv_bfloat162 hi = __floats2bfloat162_rn(a, b);
                            const __nv_bfloat162 lo = __floats2bfloat162_rn(a - __low2float(hi), b - __high2float(hi));
                            hw[w2] = *reinterpret_cast<const uint32_t *>(&hi);
                            lw[w2] = *reinterpret_cast<const uint32_t *>(&lo);
                        }
                        const int eh = hbase + c8 * 8, el = C::LO + hbase + c8 * 8;
                        *reinterpret_cast<uint4 *>(prow + (eh / HALF_VALS) * C::P_ATOMB + ((((eh % HALF_VALS) >> 3) ^ swz) << 4)) =
                            make_uint4(hw[0], hw[1], hw[2], hw[3]);
                        *reinterpret_cast<uint4 *>(prow + (el / HALF_VALS) * C::P_ATOMB + ((((el % HALF_VALS) >> 3) ^ swz) << 4)) =
                            make_uint4(lw[0], lw[1], lw[2], lw[3]);
                    }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->p_full[j2]);

                if (jj > 0) {
                    // O(i-1) was computed against the previous max; fold it in and move the
                    // running sum to the current max.
                    const int t = i - 1, jt = t & 1;
                    if (!wait_bounded(&sm->o_full[jt], (t >> 1) & 1, abort_flag, budget)) {
                        bad = true;
                        continue;
                    }
                    tc_fence_after_sync();
                    const uint32_t obase = tmem + lane_addr + C::O_COL + jt * C::OB + hbase;
                    if constexpr (C::LO == 8) {
                        uint32_t v[16];  // high parts in columns 0..7, low parts in 8..15
                        tmem_ld16(obase, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < NHW; ++e)
                            O[e] = (O[e] + (__uint_as_float(v[e]) + __uint_as_float(v[8 + e]))) * alpha[e];
                    } else {
#pragma unroll
                        for (int c = 0; c < NHW; c += 16) {
                            uint32_t hi[16], lo[16];
                            tmem_ld16(obase + c, hi);
                            tmem_ld16(obase + C::LO + c, lo);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (c + e < NHW)
                                    O[c + e] = (O[c + e] + (__uint_as_float(hi[e]) + __uint_as_float(lo[e]))) * alpha[c + e];
                        }
                    }
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->o_empty[jt]);
                }
            }
            if (!ok) break;
            if (!bad && wait_bounded(&sm->o_full[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, budget)) {
                // Last tile of the piece: its O is already relative to the final max.
                const int jt = (i - 1) & 1;
                tc_fence_after_sync();
                const uint32_t obase = tmem + lane_addr + C::O_COL + jt * C::OB + hbase;
                if constexpr (C::LO == 8) {
                    uint32_t v[16];  // high parts in columns 0..7, low parts in 8..15
                    tmem_ld16(obase, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < NHW; ++e) O[e] += __uint_as_float(v[e]) + __uint_as_float(v[8 + e]);
                } else {
#pragma unroll
                    for (int c = 0; c < NHW; c += 16) {
                        uint32_t hi[16], lo[16];
                        tmem_ld16(obase + c, hi);
                        tmem_ld16(obase + C::LO + c, lo);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (c + e < NHW) O[c + e] += __uint_as_float(hi[e]) + __uint_as_float(lo[e]);
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->o_empty[jt]);
            } else {
                bad = true;
            }
            // Sum of the softmax numerators over the 128 rows of every tile of the piece.
#pragma unroll
            for (int h = 0; h < NHW; ++h) {
                const float sum = warp_sum_f32(l[h]);
                if (lane == 0) sm->lsum[wg][q4][h] = sum;
            }
            if (named_bar_any(bar_id, 128, bad)) {
                ok = false;
                break;
            }
            if (dcol >= 0) {
                if (sg.whole) {
#pragma unroll
                    for (int h = 0; h < NHW; ++h) {
                        const long long orow = out_row(p, sg.b, sg.kvh, sg.hb, hbase + h);
                        if (orow >= 0) {
                            const float L = sm->lsum[wg][0][h] + sm->lsum[wg][1][h] + sm->lsum[wg][2][h] + sm->lsum[wg][3][h];
                            p.out[orow * D + dcol] = O[h] / L;
                        }
                    }
                } else {
                    // slot: O [RB][D], then m [RB], then l [RB] (padding columns included)
                    float *slot = p.ws + p.slot_base +
                                  (static_cast<long long>(blockIdx.x) + sg.unit) * p.slot_floats;
#pragma unroll
                    for (int h = 0; h < NHW; ++h)
                        if (hbase + h < p.RB) slot[(hbase + h) * D + dcol] = O[h];
                    if (dcol < NHW && hbase + dcol < p.RB) {
                        const int h = dcol;
                        float m_final = -INFINITY;
#pragma unroll
                        for (int hh = 0; hh < NHW; ++hh)
                            if (hh == h) m_final = m_run[hh];
                        slot[p.RB * D + hbase + h] = m_final;
                        slot[p.RB * D + p.RB + hbase + h] = sm->lsum[wg][0][h] + sm->lsum[wg][1][h] + sm->lsum[wg][2][h] + sm->lsum[wg][3][h];
                    }
                }
            }
            // the next piece rewrites lsum only after every thread has read it, and the slot
            // is complete before the ticket warp is told
            named_bar_sync(bar_id, 128);
            if (!sg.whole) {
                if (sm_tid == 128 * wg && npart < 2) mbar_arrive(&sm->pc_full[wg][npart]);
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
static int launch_split_tc_impl(const TmaMaps &maps, const DecodeParams &p, cudaStream_t stream) {
    using C = TcCfg<D, NH>;
    auto kern = split_tc_kernel<D, NH, PAGED>;
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
    if (cudaLaunchKernelEx(&cfg, kern, maps.q, maps.k, maps.k8, maps.v, maps.v8, p) != cudaSuccess)
        return GQA_ERR_CUDA;
    return GQA_OK;
}

template <int D, bool PAGED>
static int launch_split_tc_d(const TmaMaps &maps, const DecodeParams &p, int nh, cudaStream_t stream) {
    switch (nh) {
        case 1: return launch_split_tc_impl<D, 1, PAGED>(maps, p, stream);
        case 2: return launch_split_tc_impl<D, 2, PAGED>(maps, p, stream);
        case 4: return launch_split_tc_impl<D, 4, PAGED>(maps, p, stream);
        case 8: return launch_split_tc_impl<D, 8, PAGED>(maps, p, stream);
        case 16: return launch_split_tc_impl<D, 16, PAGED>(maps, p, stream);
        default: return launch_split_tc_impl<D, 32, PAGED>(maps, p, stream);  // units have <= 32 columns
    }
}

// Query heads per unit rounded up to a power of two (the kernel's compile-time head count).
int tc_heads_bucket(int heads_per_unit) {
    int nh = 1;
    while (nh < heads_per_unit) nh <<= 1;
    return nh;
}

// Cached rows per tile of the bf16 kernel for this head dimension and unit width (TcCfg::T).
int tc_tile_rows(int d, int heads_per_unit) {
    return (d == 64 && tc_heads_bucket(heads_per_unit) <= 8) ? 256 : 128;
}

// Rows of the q TMA box: the UMMA N of S^T = K.Q^T.
int tc_q_box_rows(int heads_per_unit) {
    const int nh = tc_heads_bucket(heads_per_unit);
    return nh < 16 ? 16 : nh;
}

int launch_split_tc(const TmaMaps &maps, const DecodeParams &p, cudaStream_t stream) {
    const int nh = tc_heads_bucket(p.RB);
    if (p.block_table != nullptr)
        return p.d == 128 ? launch_split_tc_d<128, true>(maps, p, nh, stream)
                          : launch_split_tc_d<64, true>(maps, p, nh, stream);
    return p.d == 128 ? launch_split_tc_d<128, false>(maps, p, nh, stream)
                      : launch_split_tc_d<64, false>(maps, p, nh, stream);
}

}  // namespace gqa
