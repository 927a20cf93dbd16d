// Warp-per-head decode step for d_k = d_v = 128 (the head shape of every workload
// in the DeltaLog evaluation: 128 x 128 fp32 state per head).
//
// Work unit = one (slot, head), owned by ONE WARP from start to end: the warp
// forms the head's key-side replay coefficients (DeltaLog paper, Section 3.3,
// computed once per slot-head pair), streams the head's 64 KB base state, writes
// o_t and the log entry, and -- as the only owner -- commits the shared log
// metadata.  No CTA-wide barrier exists: the eight warps of a CTA work on eight
// independent heads, so one head's latencies hide behind the others.
//
// Lane l owns rows 4l..4l+3 for the key-side vectors (q, k, lbar_t, a_i,
// Lambda_i) and columns 4l..4l+3 for the value side (v, b_i, o_t, and the
// mat-vec accumulators).  The mat-vecs S^T qt and S^T kt need every row's qt/kt
// in every lane: they come from the owning lane by warp shuffle, so each lane
// accumulates its four columns over all 128 rows with no cross-lane reduction.
// Replay dot products (q^T a_i, k^T a_i) are warp butterfly sums.
//
// Base-state streaming: each warp has its own ring of NSW shared-memory stages of
// 8 KB (16 contiguous rows).  Lane 0 keeps NSW chunks in flight with
// cp.async.bulk (TMA bulk copies, mbarrier complete_tx), running ahead from one
// head into the warp's next head, whose slot id is read one head early.  A merge
// step streams the tile twice: pass 1 for the mat-vecs, pass 2 -- an L2 hit,
// the pass-1 copies ask L2 to keep the lines -- to write back the materialised
// state S_t = e^{lbar_t} Sbar + sum_i A'_i b_i^T + k b_t^T.
//
// Every wait is bounded (100 ms); a warp whose wait runs out sets
// DL_EBIT_TIMEOUT, stops, and waits (bounded again) for its own copies still in
// flight before it exits.
#pragma once

#include "dl_kernels.cuh"
#include "dl_ptx.cuh"

namespace dl {
namespace wh {

constexpr int DK = 128, DV = 128;
constexpr int CR = 16;                      // rows per chunk
constexpr int NCH = DK / CR;                // chunks per pass
constexpr int CF = CR * DV;                 // floats per chunk
constexpr uint32_t CB = CF * 4;             // 8 KB
constexpr int NW = 8;                       // warps (heads in flight) per CTA
constexpr int NTHREADS = NW * 32;
constexpr int NSW = 3;                      // stages per warp
constexpr int RPB = 4;                      // log entries per ReplayPrep load block
constexpr int MRB = CF / (DK + DV);         // entries per merge round (A' and b in one stage)
constexpr uint64_t WAIT_NS = 100000000ull;  // bound on every wait
constexpr int NB = NSW + 2;                 // mbarriers per warp: stream stages + merge re-stream
constexpr size_t SMEM = (size_t)NW * NSW * CB + (size_t)NW * NB * 8 + 16;
static_assert(NSW == 3, "the merge write-back uses stages 0-1 for the tile and stage 2 as scratch");
constexpr unsigned FULL = 0xffffffffu;

template <typename T> __device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <> __device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
    const float4 x = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
template <> __device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    v[0] = __low2float(lo); v[1] = __high2float(lo); v[2] = __low2float(hi); v[3] = __high2float(hi);
}

__device__ __forceinline__ float4 ldg4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float warp_allsum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

// One head as the warp sees it.
struct Head {
    int it;        // work item (batch row * H + head), n_items when past the end
    int s;         // slot id
    int c;         // live entries
    int st;        // 0, or the error bit that makes the head skipped
    int n;         // chunks in its stream: 0 (bad slot), 8, or 16 (merge / eager)
    int merge;     // merge step (or eager step)
    size_t head;   // (slot, layer, head) index
};

template <int DECAY, bool DELTA, typename IT>
__global__ void __launch_bounds__(NTHREADS, 1) warp_head_kernel(const KParams p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float *st = reinterpret_cast<float *>(smem) + (size_t)w * NSW * CF;
    uint64_t *fb = reinterpret_cast<uint64_t *>(smem + (size_t)NW * NSW * CB) + w * NB;
    uint64_t *pb = fb + NSW;  // merge write-back: tile re-stream through stages 0 and 1
    int *next_k = reinterpret_cast<int *>(smem + (size_t)NW * NSW * CB + (size_t)NW * NB * 8);
    if (lane == 0) {
        for (int s = 0; s < NB; ++s) ptx::mbar_init(&fb[s], 1);
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 0) *next_k = NW;  // warp w starts with the CTA's w-th head
    __syncthreads();

    const int n_items = p.batch * p.H;
    const int G = gridDim.x;
    // heads of this CTA: blockIdx.x + k * G; warps take the next k from a shared
    // counter as they finish, so a warp held up by a merge head takes fewer heads
    auto grab = [&]() -> int {
        int k = 0;
        if (lane == 0) k = atomicAdd(next_k, 1);
        k = __shfl_sync(FULL, k, 0);
        const long long it = (long long)blockIdx.x + (long long)k * G;
        return it < n_items ? (int)it : n_items;
    };
    const int E = p.E;
    const uint64_t pol_stream = ptx::policy_evict_first();
    const uint64_t pol_keep = ptx::policy_evict_last();

    // -- head metadata: slot id first (it locates the tile and lets the first
    //    chunks go out), live length after (it decides append or merge)
    auto slot_of = [&](int it) -> int { return it < n_items ? p.slots[it / p.H] : -1; };
    auto len_of = [&](const Head &hd) -> int {
        return (hd.n && p.log_len) ? p.log_len[(size_t)hd.s * p.n_layers + p.layer] : 0;
    };
    auto resolve_slot = [&](Head &hd, int it, int s) {
        hd.it = it;
        hd.s = s;
        hd.c = 0;
        hd.st = 0;
        hd.merge = 0;
        hd.head = 0;
        hd.n = 0;
        if (it >= n_items) return;
        if (s < 0 || s >= p.n_slots) { hd.st = DL_EBIT_SLOT_RANGE; return; }
        hd.head = ((size_t)s * p.n_layers + p.layer) * p.H + (it % p.H);
        hd.n = NCH;  // pass 1 never depends on the live length
    };
    auto resolve_len = [&](Head &hd, int c) {
        if (!hd.n) return;
        hd.c = c;
        if (p.eager) {
            if (hd.c != 0) hd.st = DL_EBIT_LIVE_LOG;
        } else if (hd.c < 0 || hd.c > p.L) {
            hd.st = DL_EBIT_LOG_LEN;
        } else if (!(p.auto_merge && hd.c >= p.L - 1) && hd.c >= p.L) {
            hd.st = DL_EBIT_LOG_FULL;
        }
        hd.merge = p.eager || (p.auto_merge && hd.c >= p.L - 1);
        hd.n = NCH;
    };
    // L2 warm-up of what the warp reads for a head besides its base state
    auto warm = [&](const Head &hd) {
        if (lane != 0 || hd.it >= n_items || hd.st) return;
        const int bi = hd.it / p.H, h = hd.it % p.H, gk = h / (p.H / p.Hk);
        ptx::prefetch_l2(static_cast<const IT *>(p.q) + ((size_t)bi * p.Hk + gk) * DK, DK * sizeof(IT));
        ptx::prefetch_l2(static_cast<const IT *>(p.k) + ((size_t)bi * p.Hk + gk) * DK, DK * sizeof(IT));
        ptx::prefetch_l2(static_cast<const IT *>(p.v) + ((size_t)bi * p.H + h) * DV, DV * sizeof(IT));
        if (DECAY == DL_DECAY_DIAG && !p.lam_const)
            ptx::prefetch_l2(p.lam + ((size_t)bi * p.H + h) * DK, DK * 4);
        if (hd.c > 0) ptx::prefetch_l2(p.log + hd.head * (size_t)p.L * E, (uint32_t)(hd.c * E * 4));
    };

    // -- the warp's chunk stream: positions [base, base + cur.n) belong to cur,
    //    then up to NCH pass-1 chunks of nxt (its live length may not be known yet)
    int gc = 0, gi = 0, base = 0;  // consumed / issued stream positions
    bool abort = false;
    uint32_t pph = 0u;             // merge re-stream barrier phases (bit b: barrier pb[b])
    uint32_t pb_pend = 0u;         // merge re-stream copies in flight (bit b)
    Head cur, nxt;
    const int it0 = (long long)blockIdx.x + (long long)w * G < n_items ? blockIdx.x + w * G : n_items;
    resolve_slot(cur, it0, slot_of(it0));
    int it_nxt = grab();                 // the warp's next head, and its slot id, one head early
    int s_nxt = slot_of(it_nxt);
    bool nxt_res = false;                // nxt's live length (hence merge or not) known

    auto issue_upto = [&](int limit) {
        while (gi < limit) {
            const Head *hd;
            int x;
            if (gi < base + cur.n) {
                hd = &cur;
                x = gi - base;
            } else {
                // a merge head needs its stages as scratch after pass 1: no look-ahead
                const int rel = gi - base - cur.n;
                const int nit = it_nxt;
                const bool ok = !(cur.merge && cur.st == 0) && nit < n_items && s_nxt >= 0 &&
                                s_nxt < p.n_slots && rel < NCH;
                if (!ok) break;
                if (lane == 0) {
                    const size_t hn = ((size_t)s_nxt * p.n_layers + p.layer) * p.H + (nit % p.H);
                    const int sg = gi % NSW;
                    ptx::mbar_arrive_expect_tx(&fb[sg], CB);
                    ptx::bulk_g2s(st + (size_t)sg * CF, p.state + hn * (size_t)(DK * DV) + (size_t)rel * CF,
                                  CB, &fb[sg], (nxt_res && nxt.merge) ? pol_keep : pol_stream);
                }
                ++gi;
                continue;
            }
            if (lane == 0) {
                const int sg = gi % NSW;
                ptx::mbar_arrive_expect_tx(&fb[sg], CB);
                ptx::bulk_g2s(st + (size_t)sg * CF, p.state + hd->head * (size_t)(DK * DV) + (size_t)x * CF,
                              CB, &fb[sg], hd->merge ? pol_keep : pol_stream);
            }
            ++gi;
        }
    };
    // wait for stream position gc; false when the wait ran out (warp-uniform)
    auto wait_chunk = [&]() -> bool {
        const bool ok = ptx::mbar_wait_bounded(&fb[gc % NSW], (gc / NSW) & 1, WAIT_NS);
        return __all_sync(FULL, ok);
    };
    // done reading stream position gc: free its stage and keep the ring full
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) ptx::fence_proxy_async_smem();
        ++gc;
        issue_upto(gc + NSW);
    };

    issue_upto(NSW);
    resolve_len(cur, len_of(cur));
    warm(cur);
    // Finalize of the previous head, checked one head later so the atomic's round
    // trip overlaps the next head's work
    int fin_old = -1, fin_len = 0;
    size_t fin_sl = 0;
    auto finish_commit = [&]() {
        if (lane == 0 && fin_old == p.H - 1) {
            p.log_len[fin_sl] = fin_len;
            p.arrive[fin_sl] = 0;
        }
        fin_old = -1;
    };

    while (cur.it < n_items) {
        // the next head: slot id read one head ago; its live length is loaded now
        // and looked at after this head's pass 1
        resolve_slot(nxt, it_nxt, s_nxt);
        nxt_res = false;
        const int c_nxt = len_of(nxt);
        if (cur.st && lane == 0) atomicOr(p.err, cur.st);

        if (cur.st == 0) {
            const int c = cur.c;
            const bool merge_now = cur.merge != 0;
            const int bi = cur.it / p.H, h = cur.it % p.H;
            const size_t row = (size_t)bi * p.H + h;
            const size_t sl = (size_t)cur.s * p.n_layers + p.layer;
            float *tile = p.state + cur.head * (size_t)(DK * DV);
            float *ring = p.log ? p.log + cur.head * (size_t)p.L * E : nullptr;
            const int gk = h / (p.H / p.Hk);

            // -- token, cumulative log-decay and prescale (rows 4l..4l+3)
            float q_own[4], k_own[4], v_own[4], lam[4] = {0.f, 0.f, 0.f, 0.f};
            float lp[4] = {0.f, 0.f, 0.f, 0.f};
            load4<IT>(static_cast<const IT *>(p.q) + ((size_t)bi * p.Hk + gk) * DK + 4 * lane, q_own);
            load4<IT>(static_cast<const IT *>(p.k) + ((size_t)bi * p.Hk + gk) * DK + 4 * lane, k_own);
            load4<IT>(static_cast<const IT *>(p.v) + row * DV + 4 * lane, v_own);
            float beta = 0.f;
            if (DELTA) beta = __ldg(p.beta + row);
            if (DECAY == DL_DECAY_DIAG) {
                const float4 l4 = ldg4(p.lam + (p.lam_const ? (size_t)h : row) * DK + 4 * lane);
                lam[0] = l4.x; lam[1] = l4.y; lam[2] = l4.z; lam[3] = l4.w;
                if (c > 0) {
                    const float4 p4 = ldg4(ring + (size_t)(c - 1) * E + DK + DV + 4 * lane);
                    lp[0] = p4.x; lp[1] = p4.y; lp[2] = p4.z; lp[3] = p4.w;
                }
            } else if (DECAY == DL_DECAY_SCALAR) {
                const float ls = __ldg(p.lam + (p.lam_const ? (size_t)h : row));
                const float ps = c > 0 ? __ldg(ring + (size_t)(c - 1) * E + DK + DV) : 0.f;
#pragma unroll
                for (int x = 0; x < 4; ++x) { lam[x] = ls; lp[x] = ps; }
            }
            float ell[4], e_own[4], qt[4], kt[4];
            float kq = 0.f;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                ell[x] = lp[x] + lam[x];
                e_own[x] = DECAY == DL_DECAY_NONE ? 1.f : expf(ell[x]);
                const float ek = (DELTA && p.undecayed && DECAY != DL_DECAY_NONE) ? expf(lp[x]) : e_own[x];
                qt[x] = e_own[x] * q_own[x];
                kt[x] = ek * k_own[x];
                kq = fmaf(q_own[x], k_own[x], kq);
            }
            kq = warp_allsum(kq);

            // -- ReplayPrep + value replay: Y += (q^T A'_i) b_i, (k^T A'_i) b_i, eight
            //    entries' loads in flight at a time
            float4 Yq = make_float4(0.f, 0.f, 0.f, 0.f), Yk = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int i0 = 0; i0 < c; i0 += RPB) {
                float4 A[RPB], B[RPB], Lq[RPB];
#pragma unroll
                for (int u = 0; u < RPB; ++u) {
                    if (i0 + u < c) {
                        const float *ent = ring + (size_t)(i0 + u) * E;
                        A[u] = ldg4(ent + 4 * lane);
                        B[u] = ldg4(ent + DK + 4 * lane);
                        if (DECAY == DL_DECAY_DIAG) {
                            Lq[u] = ldg4(ent + DK + DV + 4 * lane);
                        } else {
                            const float Ls = DECAY == DL_DECAY_SCALAR ? __ldg(ent + DK + DV) : 0.f;
                            Lq[u] = make_float4(Ls, Ls, Ls, Ls);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < RPB; ++u) {
                    if (i0 + u < c) {
                        const float av[4] = {A[u].x, A[u].y, A[u].z, A[u].w};
                        const float Lv[4] = {Lq[u].x, Lq[u].y, Lq[u].z, Lq[u].w};
                        float pq = 0.f, pk = 0.f;
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const float g = DECAY == DL_DECAY_NONE ? 1.f : expf(ell[x] - Lv[x]);
                            const float wq = av[x] * g;
                            pq = fmaf(wq, q_own[x], pq);
                            if (DELTA) {
                                const float wk = (p.undecayed && DECAY != DL_DECAY_NONE)
                                                     ? av[x] * expf(lp[x] - Lv[x]) : wq;
                                pk = fmaf(wk, k_own[x], pk);
                            }
                        }
                        pq = warp_allsum(pq);
                        fma4(Yq, pq, B[u]);
                        if (DELTA) {
                            pk = warp_allsum(pk);
                            fma4(Yk, pk, B[u]);
                        }
                    }
                }
            }

            // the next head's phase is known from here on (its chunks' L2 policy)
            resolve_len(nxt, c_nxt);
            nxt_res = true;
            warm(nxt);

            // -- AppendDecode pass 1: y_q = Sbar^T qt, y_k = Sbar^T kt (columns 4l..4l+3)
            for (int cx = 0; cx < NCH; ++cx) {
                if (!wait_chunk()) { abort = true; break; }
                const float *sb = st + (size_t)(gc % NSW) * CF;
#pragma unroll
                for (int rr = 0; rr < CR; ++rr) {
                    const float4 S = reinterpret_cast<const float4 *>(sb + rr * DV)[lane];
                    const int src = 4 * cx + (rr >> 2);
                    fma4(Yq, __shfl_sync(FULL, qt[rr & 3], src), S);
                    if (DELTA) fma4(Yk, __shfl_sync(FULL, kt[rr & 3], src), S);
                }
                release();
            }
            if (abort) break;

            finish_commit();

            // -- b_t, o_t, and the append (entry c) or the merge-step write-back
            const float yq[4] = {Yq.x, Yq.y, Yq.z, Yq.w}, yk[4] = {Yk.x, Yk.y, Yk.z, Yk.w};
            float bt[4], o[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                bt[x] = DELTA ? beta * (v_own[x] - yk[x]) : v_own[x];
                o[x] = fmaf(bt[x], kq, yq[x]);
            }
            const float4 bt4 = make_float4(bt[0], bt[1], bt[2], bt[3]);
            if (p.want_out)
                *reinterpret_cast<float4 *>(p.out + row * DV + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
            if (!merge_now) {
                float *ent = ring + (size_t)c * E;
                *reinterpret_cast<float4 *>(ent + DK + 4 * lane) = bt4;
                *reinterpret_cast<float4 *>(ent + 4 * lane) = make_float4(k_own[0], k_own[1], k_own[2], k_own[3]);
                if (DECAY == DL_DECAY_DIAG)
                    *reinterpret_cast<float4 *>(ent + DK + DV + 4 * lane) = make_float4(ell[0], ell[1], ell[2], ell[3]);
                if (DECAY == DL_DECAY_SCALAR && lane == 0) ent[DK + DV] = ell[0];
            } else {
                // Merge step: S_t = e^{lbar_t} (.) Sbar + sum_{i<=c} A'_i b_i^T, entry c being
                // the token (A'_c = k, b_c = b_t).  Pass 1 left every stage idle (no
                // look-ahead past a merge head).  Per round of up to MRB entries, stage 2
                // holds A' (this lane's rows) and b (its columns); the tile is re-streamed
                // from L2 through stages 0/1 (Sbar in the first round, the previous round's
                // partial sums after that) and rewritten row block by row block.
                float *As = st + (size_t)2 * CF, *Bs = As + (size_t)MRB * DK;
                const int ne = c + 1;
                for (int g0 = 0; g0 < ne && !abort; g0 += MRB) {
                    const int g1 = min(ne, g0 + MRB);
                    const bool first = g0 == 0, last = g1 == ne;
                    auto issue_s = [&](int cx) {
                        if (lane == 0) {
                            uint64_t *bar = &pb[cx & 1];
                            ptx::mbar_arrive_expect_tx(bar, CB);
                            ptx::bulk_g2s(st + (size_t)(cx & 1) * CF, tile + (size_t)cx * CF, CB, bar,
                                          last ? pol_stream : pol_keep);
                        }
                        pb_pend |= 1u << (cx & 1);
                    };
                    issue_s(0);
                    issue_s(1);
                    for (int i0 = g0; i0 < g1; i0 += RPB) {
                        float4 A[RPB], B[RPB], Lq[RPB];
#pragma unroll
                        for (int u = 0; u < RPB; ++u) {
                            const int i = i0 + u;
                            if (i < g1 && i < c) {
                                const float *ent = ring + (size_t)i * E;
                                A[u] = ldg4(ent + 4 * lane);
                                B[u] = ldg4(ent + DK + 4 * lane);
                                if (DECAY == DL_DECAY_DIAG) {
                                    Lq[u] = ldg4(ent + DK + DV + 4 * lane);
                                } else {
                                    const float Ls = DECAY == DL_DECAY_SCALAR ? __ldg(ent + DK + DV) : 0.f;
                                    Lq[u] = make_float4(Ls, Ls, Ls, Ls);
                                }
                            }
                        }
#pragma unroll
                        for (int u = 0; u < RPB; ++u) {
                            const int i = i0 + u;
                            if (i >= g1) continue;
                            float4 aw, bw;
                            if (i < c) {
                                const float av[4] = {A[u].x, A[u].y, A[u].z, A[u].w};
                                const float Lv[4] = {Lq[u].x, Lq[u].y, Lq[u].z, Lq[u].w};
                                float w4[4];
#pragma unroll
                                for (int x = 0; x < 4; ++x)
                                    w4[x] = DECAY == DL_DECAY_NONE ? av[x] : av[x] * expf(ell[x] - Lv[x]);
                                aw = make_float4(w4[0], w4[1], w4[2], w4[3]);
                                bw = B[u];
                            } else {
                                aw = make_float4(k_own[0], k_own[1], k_own[2], k_own[3]);
                                bw = bt4;
                            }
                            reinterpret_cast<float4 *>(As + (size_t)(i - g0) * DK)[lane] = aw;
                            reinterpret_cast<float4 *>(Bs + (size_t)(i - g0) * DV)[lane] = bw;
                        }
                    }
                    __syncwarp();
                    for (int cx = 0; cx < NCH; ++cx) {
                        const uint32_t bb = cx & 1;
                        const bool ok = ptx::mbar_wait_bounded(&pb[bb], (pph >> bb) & 1u, WAIT_NS);
                        if (!__all_sync(FULL, ok)) { abort = true; break; }
                        pph ^= 1u << bb;
                        pb_pend &= ~(1u << bb);
                        const float *sb = st + (size_t)(cx & 1) * CF;
                        float4 acc[CR];
#pragma unroll
                        for (int rr = 0; rr < CR; ++rr) {
                            const float4 S = reinterpret_cast<const float4 *>(sb + rr * DV)[lane];
                            if (first) {
                                const float e = __shfl_sync(FULL, e_own[rr & 3], 4 * cx + (rr >> 2));
                                acc[rr] = make_float4(S.x * e, S.y * e, S.z * e, S.w * e);
                            } else {
                                acc[rr] = S;
                            }
                        }
                        for (int j = 0; j < g1 - g0; ++j) {
                            const float4 b4 = reinterpret_cast<const float4 *>(Bs + (size_t)j * DV)[lane];
                            const float *arow = As + (size_t)j * DK + cx * CR;
#pragma unroll
                            for (int rr = 0; rr < CR; ++rr) fma4(acc[rr], arow[rr], b4);
                        }
#pragma unroll
                        for (int rr = 0; rr < CR; ++rr) {
                            float4 *dst = reinterpret_cast<float4 *>(tile + (size_t)(cx * CR + rr) * DV) + lane;
                            if (last) __stcs(dst, acc[rr]);
                            else *dst = acc[rr];
                        }
                        __syncwarp();
                        if (lane == 0) ptx::fence_proxy_async_smem();
                        if (cx + 2 < NCH) issue_s(cx + 2);
                    }
                    // the next round's bulk copies re-read what this round wrote
                    ptx::fence_proxy_async_global();
                    __syncwarp();
                }
                if (abort) break;
                // the stages go back to the head stream
                if (lane == 0) ptx::fence_proxy_async_smem();
            }

            // -- Finalize: the last unit of the (slot, layer) commits the live length
            //    (the atomic is issued now, its result looked at one head later)
            if (!p.eager) {
                if (lane == 0) fin_old = atomicAdd(p.arrive + sl, 1);
                fin_sl = sl;
                fin_len = merge_now ? 0 : c + 1;
            }
        } else {
            // skipped head: consume (and ignore) the chunks that were streamed for it
            for (int x = 0; x < cur.n; ++x) {
                if (!wait_chunk()) { abort = true; break; }
                release();
            }
            if (abort) break;
            resolve_len(nxt, c_nxt);
            nxt_res = true;
            warm(nxt);
            finish_commit();
        }

        // advance: nxt becomes cur; take the head after it and read its slot id
        base += cur.n;
        cur = nxt;
        it_nxt = grab();
        s_nxt = slot_of(it_nxt);
        nxt_res = false;
        issue_upto(gc + NSW);
    }
    finish_commit();

    if (abort) {
        if (lane == 0) atomicOr(p.err, DL_EBIT_TIMEOUT);
        // no bulk copy may land in shared memory after the CTA has exited
        for (; gc < gi; ++gc) ptx::mbar_wait_bounded(&fb[gc % NSW], (gc / NSW) & 1, WAIT_NS);
        for (int b2 = 0; b2 < 2; ++b2)
            if ((pb_pend >> b2) & 1u) ptx::mbar_wait_bounded(&pb[b2], (pph >> b2) & 1u, WAIT_NS);
    }
}

}  // namespace wh
}  // namespace dl
