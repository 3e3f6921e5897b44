// Work partition and piece merge shared by the split-KV kernels.
//
// The decode work is cut into tiles of T cached rows.  A "unit" is one (sequence b, key/value
// head j, block of up to 32 query heads of j's group); a unit has ceil(n_b / T) tiles.  Units
// are ordered b-major, and the tiles of all units form one line of `total` tiles.  The split
// kernel runs G persistent CTAs and CTA i takes the contiguous tile range
//     [floor(i * total / G), floor((i + 1) * total / G)),
// so every CTA streams the same number of tiles (to within one) whatever the length mix.  A
// CTA range may cut a unit; each (CTA, unit) piece produces a partial result in workspace
// slot (CTA index + unit index), which is unique because both indices grow along the line.
// A unit covered by a single piece is finished by that CTA; a unit cut into pieces is merged
// inside the same kernel (piece merge, below).  Every kernel derives the same partition from
// seq_lens on the device, so the host never needs the lengths.
#pragma once

#include <cstdint>

#include "device.cuh"
#include "gqa.h"

namespace gqa {

struct DecodeParams {
    const int32_t *seq_lens;  // [B] rows attended per sequence
    float *out;               // [B][H_q][d]
    float *ws;                // workspace: per-unit piece counters, then partial slots
    int32_t *status;          // device status word or nullptr
    int B, H_q, H_kv, d, L_max;
    int r;     // query heads per key/value head
    int Q;     // query tokens per sequence (1, or several for speculative verification)
    int rb;    // query heads per unit and token; a unit's columns are (token j, head h') pairs
    int RB;    // columns per unit = Q * rb (<= 32), column index j * rb + h'
    int HB;    // units per key/value head = ceil(r / rb)
    int q_box_bytes;  // bytes of the q tile of one unit (bf16 path)
    int UB;    // units per sequence = H_kv * HB
    int T;     // cached rows per tile
    int G;     // CTAs of the split kernel
    int window;  // > 0: attend only the last `window` rows of each sequence; 0: all rows
    // Paged cache (block_table != nullptr): row t of sequence b is row t % page_size of page
    // block_table[b * max_pages + t / page_size] of a pool of n_pages pages; L_max is then
    // max_pages * page_size.
    const int32_t *block_table;
    int max_pages, page_size, n_pages;
    // FP8 (e4m3) cache: a code of key/value head g stands for value(code) * k_scale[g] (K)
    // or value(code) * v_scale[g] (V); nullptr for 16- and 32-bit caches.
    const float *k_scale, *v_scale;
    // Append fused into the decode (gqa_kv_append_decode): k_new / v_new [B][H_kv][d] go to row
    // seq_lens[b] of the cache, which the decode then attends (n_b = seq_lens[b] + 1); the
    // lengths after the append are written to lens_out (never to seq_lens).  append = 0: none.
    const void *k_new, *v_new;
    void *k_cache, *v_cache;  // [B][L_max][H_kv][d], for the appended rows
    int32_t *lens_out;
    int append;
    int32_t *cnt;                     // [units] pieces of each unit finished in this call (0 between calls)
    float scale_log2;                 // softmax scale * log2(e)
    unsigned long long wait_ns;       // bound of every pipeline wait
    long long slot_floats;            // RB * (d + 2) rounded up to a multiple of 4
    long long slot_base;              // offset of the first partial slot in ws, in floats
};

// Row of out [B*Q][H_q] that unit column hh (token hh / rb, head hh % rb) writes, or -1 for a
// padding column (past the group's heads in the last head block).
__device__ __forceinline__ long long out_row(const DecodeParams &p, int b, int kvh, int hb, int hh) {
    const int j = hh / p.rb, hp = hh - j * p.rb;
    const int nhb = min(p.rb, p.r - hb * p.rb);
    if (j >= p.Q || hp >= nhb) return -1;
    return (static_cast<long long>(b) * p.Q + j) * p.H_q + kvh * p.r + hb * p.rb + hp;
}

// Rows a sequence of length n may attend: n, or 0 when n is out of range -- negative, past
// L_max, or (several query tokens) shorter than the Q tokens that must be in the cache.
__device__ __forceinline__ int valid_len(int n, int L_max, int Q) {
    return (n < 0 || n > L_max || (Q > 1 && n < Q)) ? 0 : n;
}

__device__ __forceinline__ int tiles_of(int n, int T) { return (n + T - 1) / T; }

// Does a fused append take place for a sequence whose length before it is `raw`?  Only when
// the row fits: 0 <= raw < L_max (gqa_kv_append refuses the others the same way).
__device__ __forceinline__ bool append_fits(int raw, int L_max) { return raw >= 0 && raw < L_max; }

// Rows sequence b is asked to attend: seq_lens[b], plus the appended row under a fused append.
__device__ __forceinline__ int asked_len(const DecodeParams &p, int b, bool *appended = nullptr) {
    const int raw = p.seq_lens[b];
    const bool app = p.append && append_fits(raw, p.L_max);
    if (appended != nullptr) *appended = app;
    return app ? raw + 1 : raw;
}

// First attended row of a sequence with n rows: n - window under a sliding window, else 0.
__device__ __forceinline__ int first_row(int n, int window) {
    return (window > 0 && n > window) ? n - window : 0;
}

// Tiles of a sequence with (valid) length n.
__device__ __forceinline__ int seq_tiles(int n, const DecodeParams &p) {
    return tiles_of(n - first_row(n, p.window), p.T);
}

// a / b for a >= 0, b > 0: a 32-bit division whenever both fit in 32 bits (the 64-bit one is
// a long emulated sequence, and the partition arithmetic sits on every CTA's start-up path).
__device__ __forceinline__ long long udiv(long long a, long long b) {
    if (((a | b) >> 32) == 0) return static_cast<unsigned>(a) / static_cast<unsigned>(b);
    return a / b;
}

__device__ __forceinline__ long long cta_range_begin(long long i, long long total, long long G) {
    return udiv(i * total, G);
}

// The CTA whose range holds tile t (the largest i with begin(i) <= t).
__device__ __forceinline__ long long cta_of_tile(long long t, long long total, long long G) {
    return udiv((t + 1) * G - 1, total);
}

__device__ __forceinline__ long long warp_incl_scan(long long v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long u = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

struct CtaRange {
    long long begin, end, total;
    int b0;          // first sequence with a tile in [begin, end) (valid when begin < end)
    long long off0;  // first tile of sequence b0 on the line
    int bl;          // sequence holding the range's last tile end - 1
    long long offl;  // first tile of sequence bl on the line
};

// Whole warp: total tiles, this CTA's range and where it starts.  When `flag_range` is set,
// lengths outside [0, L_max] set GQA_STATUS_SEQLEN_RANGE.
__device__ inline CtaRange locate_cta_range(const DecodeParams &p, int cta, int lane, bool flag_range) {
    long long run = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        int n = 0;
        if (b < p.B) {
            bool app = false;
            const int asked = asked_len(p, b, &app);
            n = valid_len(asked, p.L_max, p.Q);
            if (flag_range) {
                if (n != asked && p.status != nullptr) atomicOr(p.status, GQA_STATUS_SEQLEN_RANGE);
                if (p.append && !app && p.status != nullptr) atomicOr(p.status, GQA_STATUS_APPEND_OVERFLOW);
                if (p.append) p.lens_out[b] = asked;
            }
        }
        const long long v = static_cast<long long>(seq_tiles(n, p)) * p.UB;
        const long long incl = warp_incl_scan(v, lane);
        run += __shfl_sync(kFullMask, incl, 31);
    }
    CtaRange cr;
    cr.total = run;
    cr.begin = cta_range_begin(cta, run, p.G);
    cr.end = cta_range_begin(cta + 1, run, p.G);
    cr.b0 = 0;
    cr.off0 = 0;
    cr.bl = 0;
    cr.offl = 0;
    if (cr.begin >= cr.end) return cr;
    long long off = 0;
    bool found0 = false;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        const int n = b < p.B ? valid_len(asked_len(p, b), p.L_max, p.Q) : 0;
        const long long v = static_cast<long long>(seq_tiles(n, p)) * p.UB;
        const long long incl = warp_incl_scan(v, lane);
        const long long excl = incl - v;
        const uint32_t m0 = __ballot_sync(kFullMask, v > 0 && off + excl <= cr.begin && cr.begin < off + incl);
        if (!found0 && m0 != 0) {
            const int l = __ffs(m0) - 1;
            cr.b0 = base + l;
            cr.off0 = off + __shfl_sync(kFullMask, excl, l);
            found0 = true;
        }
        const uint32_t ml = __ballot_sync(kFullMask, v > 0 && off + excl <= cr.end - 1 && cr.end - 1 < off + incl);
        if (ml != 0) {
            const int l = __ffs(ml) - 1;
            cr.bl = base + l;
            cr.offl = off + __shfl_sync(kFullMask, excl, l);
            return cr;
        }
        off += __shfl_sync(kFullMask, incl, 31);
    }
    return cr;  // unreachable when begin < total
}

// One CTA-range piece of one unit.
struct Segment {
    int b, kvh, hb;  // sequence, key/value head, block of query heads
    int j0, len;     // first tile (within the unit) and number of tiles of the piece
    int n;           // rows in sequence b
    int first;       // first attended row (0 unless a sliding window cuts the front)
    int unit;        // unit index b * UB + (kvh * HB + hb)
    bool whole;      // the piece is the entire unit
    bool appended;   // a fused append writes row n - 1 of the sequence
    int nt;          // tiles of the unit
    long long uoff;  // line position of the unit's first tile

    // Tile (within the unit) that the piece computes jj-th.  A piece that ends the unit takes
    // the unit's last tile first: that tile is the one a fused append patches and the one that
    // is cut short when the length is not a multiple of the tile, and its extra latency then
    // hides behind the loads of the tiles after it instead of ending the CTA's work.  Online
    // softmax does not depend on the order; every kernel and the page cursor use this one map.
    __device__ __forceinline__ int tile(int jj) const {
        if (j0 + len == nt && len > 1) return jj == 0 ? nt - 1 : j0 + jj - 1;
        return j0 + jj;
    }
    // The piece's jj-th tile is the unit's last one.
    __device__ __forceinline__ bool last_tile(int jj) const {
        return j0 + len == nt && (len > 1 ? jj == 0 : true);
    }
};

// Walks the segments of one CTA range: its last segment first (when the range has more than
// one), then the others in line order.  The last segment usually starts a unit that the next
// CTA finishes with its first segment, so both pieces of that unit are computed early and its
// merge happens early too, not at the end of the kernel.  Each role of the CTA runs its own
// walker; all of them see the same sequence of segments.
struct SegmentWalker {
    const int32_t *lens;
    int B, UB, HB, L_max, T, window, Q, append;
    int b, n, nt;
    bool app;         // sequence b takes a fused append
    long long off, t, end;
    bool last_first;  // the range's last segment is still to be returned first
    int bl, nl, ntl, kl;
    bool appl;
    long long offl, tl, endl;

    // Rows sequence bb attends (and whether a fused append writes its last one).
    __device__ int rows_of(int bb, bool &a) const {
        const int raw = lens[bb];
        a = append && append_fits(raw, L_max);
        return valid_len(a ? raw + 1 : raw, L_max, Q);
    }

    __device__ void init(const DecodeParams &p, const CtaRange &cr) {
        lens = p.seq_lens;
        B = p.B;
        UB = p.UB;
        HB = p.HB;
        L_max = p.L_max;
        T = p.T;
        window = p.window;
        Q = p.Q;
        append = p.append;
        t = cr.begin;
        end = cr.end;
        b = cr.b0;
        off = cr.off0;
        last_first = false;
        app = appl = false;
        if (t < end) {
            n = rows_of(b, app);
            nt = tiles_of(n - first_row(n, window), T);
            bl = cr.bl;
            offl = cr.offl;
            nl = rows_of(bl, appl);
            ntl = tiles_of(nl - first_row(nl, window), T);
            kl = static_cast<int>(udiv(end - 1 - offl, ntl));
            const long long uoffl = offl + static_cast<long long>(kl) * ntl;
            if (uoffl > t) {  // more than one segment: the last one is [uoffl, end)
                last_first = true;
                tl = uoffl;
                endl = end;
                end = uoffl;
            }
        } else {
            n = 0;
            nt = 0;
        }
    }

    __device__ bool next(Segment &s) {
        if (last_first) {
            last_first = false;
            const int len = static_cast<int>(endl - tl);
            s.b = bl;
            s.kvh = kl / HB;
            s.hb = kl - s.kvh * HB;
            s.j0 = 0;
            s.len = len;
            s.n = nl;
            s.first = first_row(nl, window);
            s.unit = bl * UB + kl;
            s.nt = ntl;
            s.uoff = tl;
            s.whole = len == ntl;
            s.appended = appl;
            return true;
        }
        if (t >= end) return false;
        while (t >= off + static_cast<long long>(nt) * UB) {
            off += static_cast<long long>(nt) * UB;
            if (++b >= B) {  // cannot happen while t < total; never read past seq_lens[B-1]
                t = end;
                return false;
            }
            n = rows_of(b, app);
            nt = tiles_of(n - first_row(n, window), T);
        }
        const long long rel = t - off;
        const int k = static_cast<int>(udiv(rel, nt));
        const int j0 = static_cast<int>(rel - static_cast<long long>(k) * nt);
        const long long left = end - t;
        const int len = static_cast<int>(left < nt - j0 ? left : nt - j0);
        s.b = b;
        s.kvh = k / HB;
        s.hb = k - s.kvh * HB;
        s.j0 = j0;
        s.len = len;
        s.n = n;
        s.first = first_row(n, window);
        s.unit = b * UB + k;
        s.nt = nt;
        s.uoff = off + static_cast<long long>(k) * nt;
        s.whole = (j0 == 0 && len == nt);
        s.appended = app;
        t += len;
        return true;
    }
};

// ---------------------------------------------------------------------- piece merge
// A unit cut into several pieces (by CTA ranges) is merged by the CTA that finishes its last
// piece: every piece stores its partial (o, m, l) in its slot, fences it, and takes a ticket
// from the unit's counter; the CTA holding the last ticket merges all slots -- the log-sum-exp
// combine below -- writes the unit's output and puts the counter back to zero.
//
// A piece c of a unit holds, per column, the unnormalised sum o_c = sum_t 2^(x_t - m_c) v_t,
// its reference m_c (log2 units) and l_c = sum_t 2^(x_t - m_c).  Softmax is a ratio of sums of
// exponentials, so the pieces merge exactly:
//     M = max_c m_c,   out = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
// The pages state the blockwise idea (split a long sequence into blocks, compute them
// independently, merge: "GQA注意力机制", section 4.2); the merge rule is this softmax algebra.

// CTAs in [c0, c1] whose ranges hold tiles of the unit at [uoff, uoff + nt); with fewer tiles
// than CTAs some ranges are empty and hold no piece.
__device__ __forceinline__ int unit_pieces(long long uoff, int nt, long long total, int G, int &c0,
                                           int &c1) {
    c0 = static_cast<int>(cta_of_tile(uoff, total, G));
    c1 = static_cast<int>(cta_of_tile(uoff + nt - 1, total, G));
    if (total >= G) return c1 - c0 + 1;
    int np = 0;
    for (int c = c0; c <= c1; ++c) np += cta_range_begin(c, total, G) < cta_range_begin(c + 1, total, G);
    return np;
}

// Counters per unit: one per group of threads that writes (and merges) its own columns.
constexpr int kPieceGroups = 4;

// A piece whose ticket was taken; only the first and the last segment of a CTA range can be
// partial pieces, so a CTA has at most two.
struct PendingPiece {
    long long uoff;
    int unit, b, kvh, hb, nt;
};

// Ticket for this group's columns of `unit`: atomic add with release semantics (the group's
// slot stores, ordered before it by the group barrier the caller just passed, become visible
// at GPU scope first) and acquire semantics (a last piece then sees every other slot).  The
// returned count is the number of pieces that finished before this one.
__device__ __forceinline__ int take_ticket(const DecodeParams &p, int unit, int group) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(p.cnt + static_cast<long long>(unit) * kPieceGroups + group)
                 : "memory");
    return old;
}

// The group (threads tid < nthr) that took a unit's last ticket merges that unit's columns
// [h0, h1): a one-pass log-sum-exp over the pieces' slots, four outputs (one float4) per
// vector, and puts the counter back to zero.
__device__ inline void merge_unit(const DecodeParams &p, const PendingPiece &u, long long total,
                                  int group, int h0, int h1, int tid, int nthr) {
    int c0, c1;
    unit_pieces(u.uoff, u.nt, total, p.G, c0, c1);
    const int nh = p.RB, d = p.d;
    h1 = min(h1, nh);
    const float *base = p.ws + p.slot_base + static_cast<long long>(u.unit) * p.slot_floats;
    const bool some_empty = total < p.G;
    const int nvec = (h1 - h0) * d / 4;
    // The non-empty pieces c0 .. c1 in line order (a CTA with an empty range holds none).
    auto next_piece = [&](int c) {
        while (c <= c1 && some_empty && cta_range_begin(c, total, p.G) >= cta_range_begin(c + 1, total, p.G)) ++c;
        return c;
    };
    // kVR vectors per thread per round.  Each piece's values for all of them are loaded at
    // once, one piece ahead of the arithmetic, so a round costs about one L2 round trip rather
    // than one per vector and piece; the arithmetic per vector is the one-pass merge in line
    // order.
    constexpr int kVR = 2;
    for (int v0 = tid; v0 < nvec; v0 += kVR * nthr) {
        int idx[kVR], hh[kVR];
        long long dst[kVR];
        float M[kVR], den[kVR];
        float4 num[kVR];
#pragma unroll
        for (int j = 0; j < kVR; ++j) {
            const int v = v0 + j * nthr;
            dst[j] = -1;
            idx[j] = 0;
            hh[j] = 0;
            M[j] = -INFINITY;
            den[j] = 0.f;
            num[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (v >= nvec) continue;
            idx[j] = h0 * d + 4 * v;
            hh[j] = idx[j] / d;
            const long long orow = out_row(p, u.b, u.kvh, u.hb, hh[j]);
            if (orow >= 0) dst[j] = orow * d + (idx[j] - hh[j] * d);
        }
        float m_n[kVR], l_n[kVR];
        float4 o_n[kVR];
        auto load = [&](int c) {
            const float *sl = base + static_cast<long long>(c) * p.slot_floats;
#pragma unroll
            for (int j = 0; j < kVR; ++j)
                if (dst[j] >= 0) {
                    m_n[j] = __ldcg(sl + nh * d + hh[j]);
                    l_n[j] = __ldcg(sl + nh * d + nh + hh[j]);
                    o_n[j] = __ldcg(reinterpret_cast<const float4 *>(sl + idx[j]));
                }
        };
        int c = next_piece(c0);
        if (c <= c1) load(c);
        while (c <= c1) {
            float m_c[kVR], l_c[kVR];
            float4 o_c[kVR];
#pragma unroll
            for (int j = 0; j < kVR; ++j) {
                m_c[j] = m_n[j];
                l_c[j] = l_n[j];
                o_c[j] = o_n[j];
            }
            c = next_piece(c + 1);
            if (c <= c1) load(c);
#pragma unroll
            for (int j = 0; j < kVR; ++j) {
                if (dst[j] < 0 || m_c[j] == -INFINITY) continue;
                if (m_c[j] > M[j]) {
                    const float sc = M[j] == -INFINITY ? 0.f : ex2_approx(M[j] - m_c[j]);
                    num[j].x *= sc; num[j].y *= sc; num[j].z *= sc; num[j].w *= sc;
                    den[j] *= sc;
                    M[j] = m_c[j];
                }
                const float wgt = ex2_approx(m_c[j] - M[j]);
                num[j].x = fmaf(wgt, o_c[j].x, num[j].x);
                num[j].y = fmaf(wgt, o_c[j].y, num[j].y);
                num[j].z = fmaf(wgt, o_c[j].z, num[j].z);
                num[j].w = fmaf(wgt, o_c[j].w, num[j].w);
                den[j] = fmaf(wgt, l_c[j], den[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kVR; ++j)
            if (dst[j] >= 0) {
                const float inv = 1.f / den[j];
                *reinterpret_cast<float4 *>(p.out + dst[j]) =
                    make_float4(num[j].x * inv, num[j].y * inv, num[j].z * inv, num[j].w * inv);
            }
    }
    if (tid == 0) p.cnt[static_cast<long long>(u.unit) * kPieceGroups + group] = 0;
}

// Bookkeeping of one group's partial pieces: record(...) right after the group barrier that
// follows a partial piece's slot stores; finish(...) after the CTA's second segment (the
// walker returns the range's two partial pieces first) and once more after its last.
struct PieceTickets {
    int n = 0;
    int done = 0;
    int ticket[2] = {0, 0};

    __device__ void record(const DecodeParams &p, const Segment &sg, int group, int tid, PendingPiece *pend) {
        if (n < 2 && tid == 0) {
            pend[n] = PendingPiece{sg.uoff, sg.unit, sg.b, sg.kvh, sg.hb, sg.nt};
            ticket[n] = take_ticket(p, sg.unit, group);
        }
        ++n;
    }

    template <typename Bar>
    __device__ void finish(const DecodeParams &p, long long total, int group, int h0, int h1, int tid, int nthr,
                           PendingPiece *pend, int *flag, Bar bar) {
        for (int k = done; k < n && k < 2; ++k) {
            if (tid == 0) {
                int c0, c1;
                *flag = ticket[k] == unit_pieces(pend[k].uoff, pend[k].nt, total, p.G, c0, c1) - 1;
            }
            bar();
            if (*flag) merge_unit(p, pend[k], total, group, h0, h1, tid, nthr);
            bar();
        }
        done = n;
    }
};

// The ticket warp of a CTA.  Each group of softmax threads (NG of them, one per head slice)
// stores a partial piece's slot and arrives on pc_full[group][k] (k: the piece's place among
// the CTA's partial pieces, at most two); this warp then takes the group's ticket for the unit
// -- the atomic's release covers the slot stores the barrier made it observe, its acquire the
// other pieces' -- and reports whether it was the last one in tk_last[group][k], arriving on
// tk_done[group][k].  The softmax threads never wait on the atomic; they merge the units
// reported to them (merge_reported) with all their threads.
template <int NG>
__device__ void run_ticket_warp(const DecodeParams &p, const CtaRange &cr, uint64_t (*pc_full)[2],
                                uint64_t (*tk_done)[2], int (*tk_last)[2], int lane,
                                const volatile int *abort_flag, uint64_t budget) {
    SegmentWalker w;
    w.init(p, cr);
    Segment sg;
    int k = 0;
    while (k < 2 && w.next(sg)) {
        if (sg.whole) continue;
        for (int g = 0; g < NG; ++g) {
            const bool got = wait_bounded(&pc_full[g][k], 0, abort_flag, budget);
            if (!__all_sync(kFullMask, got)) return;  // the softmax side failed; it reports it
            if (lane == 0) {
                int c0, c1;
                tk_last[g][k] = take_ticket(p, sg.unit, g) == unit_pieces(sg.uoff, sg.nt, cr.total, p.G, c0, c1) - 1;
                mbar_arrive(&tk_done[g][k]);
            }
        }
        ++k;
    }
}

// Softmax side of the ticket warp, for one group of nthr threads: the units whose last ticket
// was reported for the group's partial pieces [done, n) are merged, in order.  Non-blocking
// (block = false) it stops at the first piece whose report is not in yet; blocking it waits
// for each.  bar_any(pred) is a barrier of the group that returns whether pred held in any
// thread, so every decision is the group's.  Returns false when a blocking wait gave up.
template <typename BarAny>
__device__ bool merge_reported(const DecodeParams &p, long long total, int group, int h0, int h1, int tid,
                               int nthr, uint64_t *tk_done, const int *tk_last, const PendingPiece *pp,
                               int n, int &done, bool block, const volatile int *abort_flag,
                               uint64_t budget, BarAny bar_any) {
    for (; done < n && done < 2; ++done) {
        const bool got = block ? wait_bounded(&tk_done[done], 0, abort_flag, budget) : mbar_test_wait(&tk_done[done], 0);
        if (bar_any(!got)) return !block;
        if (tk_last[done]) merge_unit(p, pp[done], total, group, h0, h1, tid, nthr);
    }
    return true;
}

// Units with no rows (a sequence of length 0, or one refused as out of range) get zero
// output; CTA `cta` of G covers units cta, cta + G, ...
__device__ inline void zero_empty_units(const DecodeParams &p, int cta, int tid, int nthr) {
    const int units = p.B * p.UB;
    for (int u = cta; u < units; u += p.G) {
        const int b = u / p.UB;
        if (seq_tiles(valid_len(asked_len(p, b), p.L_max, p.Q), p) != 0) continue;
        const int k = u - b * p.UB;
        const int kvh = k / p.HB, hb = k - kvh * p.HB;
        for (int idx = tid; idx < p.RB * p.d; idx += nthr) {
            const long long orow = out_row(p, b, kvh, hb, idx / p.d);
            if (orow >= 0) p.out[orow * p.d + idx % p.d] = 0.f;
        }
    }
}

// Tiles ahead of the copy at which the paged producer loads page ids.
constexpr int kPageAhead = 2;

// A cursor over the tiles of a CTA's range, one tile at a time, used to look up page ids ahead
// of the tile being copied.
struct TileCursor {
    SegmentWalker w;
    Segment sg;
    int jj;
    bool live;

    __device__ void init(const DecodeParams &p, const CtaRange &cr) {
        w.init(p, cr);
        live = w.next(sg);
        jj = 0;
    }
    __device__ void advance() {
        if (live && ++jj >= sg.len) {
            live = w.next(sg);
            jj = 0;
        }
    }
    // Page holding box `box` of the current tile (boxes as the producer cuts them: T / boxr
    // boxes of min(page_size, T) rows for a full tile, 8-row boxes for a partial one); 0 past
    // the last box or the last tile.  Every box starts below the sequence's length, so the
    // block-table index stays below max_pages.
    __device__ int page_of_box(const DecodeParams &p, int T, int box) const {
        if (!live) return 0;
        const int row0 = sg.first + sg.tile(jj) * T;
        const int rows = min(T, sg.n - row0);
        const int boxr = rows == T ? min(p.page_size, T) : 8;
        const int nbox = rows == T ? T / boxr : (rows + 7) >> 3;
        if (box >= nbox) return 0;
        return __ldg(p.block_table + static_cast<long long>(sg.b) * p.max_pages + (row0 + box * boxr) / p.page_size);
    }
};

}  // namespace gqa
