// sm_100a kernels of the base + log recurrent-state decode step.
//
// Work decomposition (DeltaLog paper, Section 3.3): one CTA per
// (slot, head, value tile); the tile is the d_k x B_V slice of the head's dense
// fp32 base state.  A head's N_V = d_v / B_V tiles are adjacent in blockIdx so the
// key-side data they share (q, k, a_i, Lambda_i) is read from HBM once and hit in L2
// by the others.
//
// Inside a CTA each thread owns RPT rows x 4 columns of the tile (one 128-bit
// word per row).  A warp's load instruction covers 32/CQ whole rows of the tile
// (128 B per row at B_V = 32), so every global access is a full, aligned line.
// The tile is fetched into registers with cache-streaming 128-bit loads at the
// top of the kernel, before any metadata is read, so the HBM stream is in flight
// while the CTA computes its replay coefficients.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dl_internal.h"
#include "dl_ptx.cuh"

namespace dl {

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <int DK, int BV> struct TileShape {
    static constexpr int CQ = BV / 4;                     // 128-bit column words per row
    static constexpr int NT = (DK * BV / 32) < 32 ? 32 : (DK * BV / 32);  // 8 words/thread
    static constexpr int RG = NT / CQ;                    // row groups
    static constexpr int RPT = DK / RG;                   // rows per thread
    static constexpr int NW = NT / 32;                    // warps
    static_assert(RPT * RG == DK, "tile rows must divide evenly");
    static_assert(32 % CQ == 0 && NT % 32 == 0, "bad tile shape");
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ---- log entry access.  The layout (fp32, or compact with bf16 a_i and, without the
// delta rule, bf16 b_i) comes from KParams; Lambda_i is fp32 at p.loff either way.
__device__ __forceinline__ float4 bf16x4_to_float4(const __nv_bfloat16 *src) {
    const uint2 u = *reinterpret_cast<const uint2 *>(src);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}
// a_i[4 r4 .. 4 r4 + 3]
__device__ __forceinline__ float4 ent_a4(const KParams &p, const float *ent, int r4) {
    if (p.a16) return bf16x4_to_float4(reinterpret_cast<const __nv_bfloat16 *>(ent) + 4 * r4);
    return *reinterpret_cast<const float4 *>(ent + 4 * r4);
}
// b_i[4 c4 .. 4 c4 + 3]
__device__ __forceinline__ float4 ent_b4(const KParams &p, const float *ent, int c4) {
    if (p.b16) return bf16x4_to_float4(reinterpret_cast<const __nv_bfloat16 *>(ent + p.boff) + 4 * c4);
    return *reinterpret_cast<const float4 *>(ent + p.boff + 4 * c4);
}
__device__ __forceinline__ float ent_a(const KParams &p, const float *ent, int r) {
    return p.a16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(ent)[r]) : ent[r];
}
// the stored values are bf16 inputs (k_t, and v_t without the delta rule), so the
// conversion back to bf16 is exact
__device__ __forceinline__ void ent_put_a(const KParams &p, float *ent, int r, float v) {
    if (p.a16) reinterpret_cast<__nv_bfloat16 *>(ent)[r] = __float2bfloat16_rn(v);
    else ent[r] = v;
}
__device__ __forceinline__ void ent_put_b(const KParams &p, float *ent, int col, float v) {
    if (p.b16) reinterpret_cast<__nv_bfloat16 *>(ent + p.boff)[col] = __float2bfloat16_rn(v);
    else ent[p.boff + col] = v;
}

__device__ __forceinline__ void fma4(float4 &acc, float a, const float4 &b) {
    acc.x = fmaf(a, b.x, acc.x);
    acc.y = fmaf(a, b.y, acc.y);
    acc.z = fmaf(a, b.z, acc.z);
    acc.w = fmaf(a, b.w, acc.w);
}

// Offsets (floats) inside the dynamic shared-memory block.
struct DynLayout {
    int cq, ck, b, A;
    __device__ __forceinline__ DynLayout(int L, int bv) {
        const int L4 = (L + 3) & ~3;
        cq = 0;
        ck = L4;
        b = 2 * L4;
        A = 2 * L4 + L * bv;
    }
};

// ---------------------------------------------------------------------------
// Decode / append / eager step.
//
// For the slot's c live entries and this step's token (paper, logical-state
// equation with lbar_t = Lambda_{c-1} + lambda_t):
//   qt = e^{lbar_t} (.) q,   kt = e^{lbar_t} (.) k   (e^{Lambda_{c-1}} for the
//                                                     undecayed delta reading)
//   cq_i = sum_r a_i[r] e^{lbar_t[r] - Lambda_i[r]} q[r]        (ReplayPrep)
//   ck_i = the same with k                                      (delta rule)
//   y_q = Sbar^T qt + sum_i cq_i b_i,  y_k = Sbar^T kt + sum_i ck_i b_i
//   b_t = v (additive) | beta (v - y_k) (delta);  o_t = y_q + b_t (k . q)
// then either append (k, b_t, lbar_t) as entry c, or, on the slot's merge step
// (on every step with p.merge_every, and always in eager mode), write
//   S_t = e^{lbar_t} (.) Sbar + sum_i A'_i b_i^T + k b_t^T,  A'_i = a_i (.) e^{lbar_t - Lambda_i}.
// ---------------------------------------------------------------------------
template <int DK, int BV, int DECAY, bool DELTA, typename IT>
__global__ void __launch_bounds__(TileShape<DK, BV>::NT)
    step_kernel(const KParams p)
{
    using Sh = TileShape<DK, BV>;
    constexpr int NT = Sh::NT, CQ = Sh::CQ, RG = Sh::RG, RPT = Sh::RPT, NW = Sh::NW;

    __shared__ float s_q[DK], s_k[DK], s_qt[DK], s_kt[DK], s_ell[DK], s_ellp[DK], s_e[DK];
    __shared__ float s_red[2][NW][BV];
    __shared__ __align__(16) float s_bt[BV];
    __shared__ float s_kq;
    extern __shared__ __align__(16) float s_dyn[];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nv = p.nv;
    const int j = blockIdx.x % nv;
    const int h = (blockIdx.x / nv) % p.H;
    const int bi = blockIdx.x / (nv * p.H);
    const int dv = p.dv;

    // A CTA that leaves early still passes the two cluster barriers its tiles wait
    // at below, so a call whose tiles disagree (slots not distinct) cannot hang them.
    auto leave = [&]() {
        if (p.cl > 1) {
            cooperative_groups::this_cluster().sync();
            cooperative_groups::this_cluster().sync();
        }
    };
    const int s = p.slots[bi];
    if (s < 0 || s >= p.n_slots) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_SLOT_RANGE);
        leave();
        return;
    }
    const size_t sl = (size_t)s * p.n_layers + p.layer;
    const size_t head = sl * p.H + h;
    float *tile = p.state + head * (size_t)DK * dv + (size_t)j * BV;
    const int quad = tid % CQ, rg = tid / CQ;

    // 1. stream the base tile (read-only on append steps)
    const bool need_base = p.want_out || DELTA || p.eager || p.auto_merge;
    float4 Sr[RPT];
    if (need_base) {
#pragma unroll
        for (int m = 0; m < RPT; ++m)
            Sr[m] = __ldcs(reinterpret_cast<const float4 *>(tile + (size_t)(rg + m * RG) * dv) + quad);
    }

    // 2. live-log length and phase
    int c = 0;
    if (p.log_len) c = p.log_len[sl];
    if (p.eager) {
        if (c != 0) {
            if (tid == 0) atomicOr(p.err, DL_EBIT_LIVE_LOG);
            leave();
            return;
        }
    } else if (c < 0 || c > p.L) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_LOG_LEN);
        leave();
        return;
    }
    const bool merge_now = p.eager || (p.auto_merge && (c >= p.L - 1 || p.merge_every));
    if (!merge_now && c >= p.L) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_LOG_FULL);
        leave();
        return;
    }
    float *ring = p.log ? p.log + head * (size_t)p.L * p.E : nullptr;
    const DynLayout lay(p.L, BV);
    float *s_cq = s_dyn + lay.cq, *s_ck = s_dyn + lay.ck, *s_b = s_dyn + lay.b, *s_A = s_dyn + lay.A;
    // A merge stages the A'_i rows in shared memory, except in launches that merge
    // every step with scalar decay (RetNet, GDN): those are sized like an eager step,
    // without the A' area (on B200 the larger allocation cost about 0.4 us per
    // 32-head launch), and the rare merge of a non-empty log there (the first step
    // after the policy changes) forms A'_i in the update loop instead, with the same
    // arithmetic.  For the other decays that loop changed the registers of every
    // launch of the instantiation (per-key decay: the eager GLA B = 64 step went from
    // 26 to 33 us), so they keep the staged rows.
    constexpr bool RECOMPUTE_OK = DECAY == DL_DECAY_SCALAR;
    const bool stage_A = !(RECOMPUTE_OK && p.merge_every);

    // 3. token, cumulative log-decay, prescaled q and k
    const int g = h / (p.H / p.Hk);
    const IT *qrow = static_cast<const IT *>(p.q) + ((size_t)bi * p.Hk + g) * DK;
    const IT *krow = static_cast<const IT *>(p.k) + ((size_t)bi * p.Hk + g) * DK;
    const float *Lprev = (c > 0) ? ring + (size_t)(c - 1) * p.E + p.loff : nullptr;
    float lam_s = 0.f;
    const float *lrow = nullptr;
    if (DECAY == DL_DECAY_SCALAR) lam_s = p.lam_const ? p.lam[h] : p.lam[(size_t)bi * p.H + h];
    if (DECAY == DL_DECAY_DIAG)
        lrow = p.lam_const ? p.lam + (size_t)h * DK : p.lam + ((size_t)bi * p.H + h) * DK;
    for (int r = tid; r < DK; r += NT) {
        const float qv = to_f32(qrow[r]), kv = to_f32(krow[r]);
        float lp = 0.f, lt = 0.f, et = 1.f, ek = 1.f;
        if (DECAY == DL_DECAY_DIAG) {
            lp = Lprev ? Lprev[r] : 0.f;
            lt = lp + lrow[r];
        } else if (DECAY == DL_DECAY_SCALAR) {
            lp = Lprev ? Lprev[0] : 0.f;
            lt = lp + lam_s;
        }
        if (DECAY != DL_DECAY_NONE) {
            et = expf(lt);
            ek = (DELTA && p.undecayed) ? expf(lp) : et;
        }
        s_q[r] = qv;
        s_k[r] = kv;
        s_ell[r] = lt;
        s_ellp[r] = lp;
        s_e[r] = et;
        s_qt[r] = et * qv;
        s_kt[r] = ek * kv;
    }
    __syncthreads();

    // 4. ReplayPrep: key-side replay coefficients, one warp per log entry.  With
    //    p.cl > 1 the head's p.cl value tiles run as one thread-block cluster and
    //    tile j forms the entries of warps j*NW .. j*NW + NW-1 of each round; the
    //    tiles read the rest from one another below.
    const int cl = p.cl, cr = p.cl > 1 ? j : 0;
    // A warp takes RU of its entries per round: their loads are all in flight before
    // the first reduction, so a long log is not a chain of dependent round trips.
    constexpr int RU = 4;
    const int stride = NW * cl;
    for (int i0 = cr * NW + warp; i0 < c; i0 += stride * RU) {
        float pqv[RU], pkv[RU];
#pragma unroll
        for (int u = 0; u < RU; ++u) {
            pqv[u] = 0.f;
            pkv[u] = 0.f;
            const int i = i0 + u * stride;
            if (i >= c) continue;
            const float *ent = ring + (size_t)i * p.E;
            float fs = 1.f, fk = 1.f;
            if (DECAY == DL_DECAY_SCALAR) {
                const float Li = ent[p.loff];
                fs = expf(s_ell[0] - Li);
                fk = (DELTA && p.undecayed) ? expf(s_ellp[0] - Li) : fs;
            }
            float pq = 0.f, pk = 0.f;
            for (int r4 = lane; r4 < DK / 4; r4 += 32) {
                const float4 a4 = ent_a4(p, ent, r4);
                float4 L4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (DECAY == DL_DECAY_DIAG) L4 = *reinterpret_cast<const float4 *>(ent + p.loff + 4 * r4);
                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
                const float Lv[4] = {L4.x, L4.y, L4.z, L4.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int r = 4 * r4 + x;
                    float w, wk;
                    if (DECAY == DL_DECAY_DIAG) {
                        w = av[x] * expf(s_ell[r] - Lv[x]);
                        wk = (DELTA && p.undecayed) ? av[x] * expf(s_ellp[r] - Lv[x]) : w;
                    } else {
                        w = av[x] * fs;
                        wk = av[x] * fk;
                    }
                    pq = fmaf(w, s_q[r], pq);
                    if (DELTA) pk = fmaf(wk, s_k[r], pk);
                    if (stage_A && merge_now) s_A[i * DK + r] = w;
                }
            }
            pqv[u] = pq;
            pkv[u] = pk;
        }
#pragma unroll
        for (int u = 0; u < RU; ++u) {
            const int i = i0 + u * stride;
            if (i >= c) continue;
            const float pq = warp_sum(pqv[u]);
            const float pk = DELTA ? warp_sum(pkv[u]) : 0.f;
            if (lane == 0) {
                s_cq[i] = pq;
                s_ck[i] = pk;
            }
        }
    }
    // value-side log shard of this tile
    for (int idx = tid; idx < c * CQ; idx += NT) {
        const int i = idx / CQ, x4 = idx % CQ;
        reinterpret_cast<float4 *>(s_b + i * BV)[x4] = ent_b4(p, ring + (size_t)i * p.E, (j * BV) / 4 + x4);
    }
    if (p.want_out && warp == 0) {  // a_t . q_t for the new entry (no decay since insertion)
        float x = 0.f;
        for (int r = lane; r < DK; r += 32) x = fmaf(s_q[r], s_k[r], x);
        x = warp_sum(x);
        if (lane == 0) s_kq = x;
    }
    __syncthreads();
    if (cl > 1) {
        // coefficients (and, on a merge step, A' rows) formed by the other tiles
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        for (int i = tid; i < c; i += NT) {
            const int o = (i / NW) % cl;
            if (o != cr) {
                s_cq[i] = *cluster.map_shared_rank(s_cq + i, o);
                if (DELTA) s_ck[i] = *cluster.map_shared_rank(s_ck + i, o);
            }
        }
        if (stage_A && merge_now) {
            for (int idx = tid; idx < c * DK; idx += NT) {
                const int o = (idx / DK / NW) % cl;
                if (o != cr) s_A[idx] = *cluster.map_shared_rank(s_A + idx, o);
            }
        }
        // no tile moves on (or leaves) while another still reads its shared memory
        cluster.sync();
    }

    // 5. AppendDecode: base mat-vecs S^T qt and S^T kt over this tile
    float yq[4] = {0.f, 0.f, 0.f, 0.f}, yk[4] = {0.f, 0.f, 0.f, 0.f};
    if (need_base) {
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int r = rg + m * RG;
            const float a = s_qt[r];
            yq[0] = fmaf(Sr[m].x, a, yq[0]);
            yq[1] = fmaf(Sr[m].y, a, yq[1]);
            yq[2] = fmaf(Sr[m].z, a, yq[2]);
            yq[3] = fmaf(Sr[m].w, a, yq[3]);
            if (DELTA) {
                const float b = s_kt[r];
                yk[0] = fmaf(Sr[m].x, b, yk[0]);
                yk[1] = fmaf(Sr[m].y, b, yk[1]);
                yk[2] = fmaf(Sr[m].z, b, yk[2]);
                yk[3] = fmaf(Sr[m].w, b, yk[3]);
            }
        }
#pragma unroll
        for (int o = CQ; o < 32; o <<= 1) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                yq[x] += __shfl_xor_sync(0xffffffffu, yq[x], o);
                if (DELTA) yk[x] += __shfl_xor_sync(0xffffffffu, yk[x], o);
            }
        }
        if (lane < CQ) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                s_red[0][warp][4 * quad + x] = yq[x];
                s_red[1][warp][4 * quad + x] = yk[x];
            }
        }
    }
    __syncthreads();

    // 6. replay the value log, form b_t and o_t, append (or prepare the merge)
    if (tid < BV) {
        const int col = j * BV + tid;
        float Yq = 0.f, Yk = 0.f;
        if (need_base) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                Yq += s_red[0][w][tid];
                Yk += s_red[1][w][tid];
            }
        }
        for (int i = 0; i < c; ++i) {
            const float b = s_b[i * BV + tid];
            Yq = fmaf(b, s_cq[i], Yq);
            if (DELTA) Yk = fmaf(b, s_ck[i], Yk);
        }
        const size_t row = (size_t)bi * p.H + h;
        const float vv = to_f32(static_cast<const IT *>(p.v)[row * dv + col]);
        const float bt = DELTA ? p.beta[row] * (vv - Yk) : vv;
        if (p.want_out) p.out[row * dv + col] = fmaf(bt, s_kq, Yq);
        if (!merge_now) ent_put_b(p, ring + (size_t)c * p.E, col, bt);
        s_bt[tid] = bt;
    }
    if (!merge_now && j == 0) {  // designated writer of the shared entry fields
        float *ent = ring + (size_t)c * p.E;
        for (int r = tid; r < DK; r += NT) {
            ent_put_a(p, ent, r, s_k[r]);
            if (DECAY == DL_DECAY_DIAG) ent[p.loff + r] = s_ell[r];
        }
        if (DECAY == DL_DECAY_SCALAR && tid == 0) ent[p.loff] = s_ell[0];
    }

    // 7. merge step: write the materialised state back over the base tile
    if (merge_now) {
        __syncthreads();
        const float4 btq = reinterpret_cast<const float4 *>(s_bt)[quad];
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int r = rg + m * RG;
            const float e = s_e[r];
            Sr[m].x *= e;
            Sr[m].y *= e;
            Sr[m].z *= e;
            Sr[m].w *= e;
            fma4(Sr[m], s_k[r], btq);
        }
        for (int i = 0; i < c; ++i) {
            const float4 b4 = reinterpret_cast<const float4 *>(s_b + i * BV)[quad];
            if (!RECOMPUTE_OK || stage_A) {
#pragma unroll
                for (int m = 0; m < RPT; ++m) fma4(Sr[m], s_A[i * DK + rg + m * RG], b4);
            } else if constexpr (RECOMPUTE_OK) {
                const float *ent = ring + (size_t)i * p.E;
                const float fs = expf(s_ell[0] - ent[p.loff]);
#pragma unroll
                for (int m = 0; m < RPT; ++m) fma4(Sr[m], ent_a(p, ent, rg + m * RG) * fs, b4);
            }
        }
#pragma unroll
        for (int m = 0; m < RPT; ++m)
            __stcs(reinterpret_cast<float4 *>(tile + (size_t)(rg + m * RG) * dv) + quad, Sr[m]);
    }

    // 8. Finalize: the last CTA of this (slot, layer) commits the live length.  A merge
    //    step that started from an empty log leaves it empty: nothing to commit, and
    //    every CTA of the slot saw the same c, so none of them counts itself in.
    if (!p.eager && !(merge_now && c == 0)) {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const int total = p.H * nv;
            const int old = atomicAdd(p.arrive + sl, 1);
            if (old == total - 1) {
                p.log_len[sl] = merge_now ? 0 : c + 1;
                p.arrive[sl] = 0;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Merge / materialise: Sbar' = e^{lbar} (.) Sbar + sum_{i<c} A'_i b_i^T with
// lbar = Lambda_{c-1}, A'_i = a_i (.) e^{lbar - Lambda_i}.  Merge writes Sbar' over
// the base and resets the live length; materialise writes it to dense_out.
// ---------------------------------------------------------------------------
template <int DK, int BV, int DECAY>
__global__ void __launch_bounds__(TileShape<DK, BV>::NT)
    merge_kernel(const KParams p, const int materialize)
{
    using Sh = TileShape<DK, BV>;
    constexpr int NT = Sh::NT, CQ = Sh::CQ, RG = Sh::RG, RPT = Sh::RPT;

    __shared__ float s_e[DK];
    extern __shared__ __align__(16) float s_dyn[];

    const int tid = threadIdx.x;
    const int nv = p.nv;
    const int j = blockIdx.x % nv;
    const int h = (blockIdx.x / nv) % p.H;
    const int bi = blockIdx.x / (nv * p.H);
    const int dv = p.dv;

    const int s = p.slots[bi];
    if (s < 0 || s >= p.n_slots) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_SLOT_RANGE);
        return;
    }
    const size_t sl = (size_t)s * p.n_layers + p.layer;
    const size_t head = sl * p.H + h;
    float *tile = p.state + head * (size_t)DK * dv + (size_t)j * BV;
    const int quad = tid % CQ, rg = tid / CQ;

    const int c = p.log_len[sl];
    if (c < 0 || c > p.L) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_LOG_LEN);
        return;
    }
    if (!materialize && c == 0) return;  // nothing to fold; live length stays 0

    float4 Sr[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        Sr[m] = __ldcs(reinterpret_cast<const float4 *>(tile + (size_t)(rg + m * RG) * dv) + quad);

    const float *ring = p.log + head * (size_t)p.L * p.E;
    const DynLayout lay(p.L, BV);
    float *s_b = s_dyn + lay.b, *s_A = s_dyn + lay.A;
    const float *Lbar = (c > 0) ? ring + (size_t)(c - 1) * p.E + p.loff : nullptr;

    for (int r = tid; r < DK; r += NT) {
        float e = 1.f;
        if (DECAY == DL_DECAY_DIAG && Lbar) e = expf(Lbar[r]);
        if (DECAY == DL_DECAY_SCALAR && Lbar) e = expf(Lbar[0]);
        s_e[r] = e;
    }
    for (int idx = tid; idx < c * DK; idx += NT) {
        const int i = idx / DK, r = idx % DK;
        const float *ent = ring + (size_t)i * p.E;
        float w = ent_a(p, ent, r);
        if (DECAY == DL_DECAY_DIAG) w *= expf(Lbar[r] - ent[p.loff + r]);
        if (DECAY == DL_DECAY_SCALAR) w *= expf(Lbar[0] - ent[p.loff]);
        s_A[idx] = w;
    }
    for (int idx = tid; idx < c * CQ; idx += NT) {
        const int i = idx / CQ, x4 = idx % CQ;
        reinterpret_cast<float4 *>(s_b + i * BV)[x4] = ent_b4(p, ring + (size_t)i * p.E, (j * BV) / 4 + x4);
    }
    __syncthreads();

#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const float e = s_e[rg + m * RG];
        Sr[m].x *= e;
        Sr[m].y *= e;
        Sr[m].z *= e;
        Sr[m].w *= e;
    }
    for (int i = 0; i < c; ++i) {
        const float4 b4 = reinterpret_cast<const float4 *>(s_b + i * BV)[quad];
#pragma unroll
        for (int m = 0; m < RPT; ++m) fma4(Sr[m], s_A[i * DK + rg + m * RG], b4);
    }
    float *dst = materialize
                     ? p.dense_out + ((size_t)bi * p.H + h) * (size_t)DK * dv + (size_t)j * BV
                     : tile;
#pragma unroll
    for (int m = 0; m < RPT; ++m)
        __stcs(reinterpret_cast<float4 *>(dst + (size_t)(rg + m * RG) * dv) + quad, Sr[m]);

    if (!materialize) {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const int old = atomicAdd(p.arrive + sl, 1);
            if (old == p.H * nv - 1) {
                p.log_len[sl] = 0;
                p.arrive[sl] = 0;
            }
        }
    }
}

}  // namespace dl

namespace dl {

// ---------------------------------------------------------------------------
// Merge / materialise of whole 128 x 128 heads (DeltaLog paper, Section 3.3,
// Merge: each dense fp32 tile is rewritten once).  One CTA of eight warps owns a
// (slot, head): warp w holds rows 16w .. 16w+15 of the tile in registers (lane l
// columns 4l .. 4l+3), loaded with streaming 128-bit loads before anything else is
// read.  The CTA forms A'^T[i][r] = a_i[r] e^{lbar[r] - Lambda_i[r]} and b_i for
// the c live entries once, in shared memory; every lane then applies
//   Sbar'[r][:] = e^{lbar[r]} Sbar[r][:] + sum_i A'^T[i][r] b_i[:]
// to its 16 rows, reading b_i (its four columns) and A'^T[i][16w..16w+15]
// (broadcast) from shared memory.  Merge writes Sbar' over the base and commits
// live length 0 (the last CTA of the slot); materialise writes it to dense_out.
// ---------------------------------------------------------------------------
constexpr int MH_NT = 256;

template <int DECAY>
__global__ void __launch_bounds__(MH_NT, 2) merge_head_kernel(const KParams p, const int materialize)
{
    constexpr int D = 128, RW = 16;
    extern __shared__ __align__(16) float s_dyn[];
    __shared__ __align__(16) float s_e[D];
    __shared__ __align__(16) float s_lb[D];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int bi = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int s = p.slots[bi];
    if (s < 0 || s >= p.n_slots) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_SLOT_RANGE);
        return;
    }
    const size_t sl = (size_t)s * p.n_layers + p.layer;
    const size_t head = sl * p.H + h;
    float *tile = p.state + head * (size_t)(D * D);
    const int c = p.log_len[sl];
    if (c < 0 || c > p.L) {
        if (tid == 0) atomicOr(p.err, DL_EBIT_LOG_LEN);
        return;
    }
    if (!materialize && c == 0) return;  // nothing to fold; live length stays 0

    // 1. the tile rows of this warp, in flight while the log is read
    float4 S[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r)
        S[r] = __ldcs(reinterpret_cast<const float4 *>(tile + (size_t)(RW * w + r) * D) + lane);

    // 2. the live entries, copied raw into shared memory with per-thread asynchronous
    //    16-byte copies as soon as c is known (lbar = Lambda_{c-1} arrives with them);
    //    then e^{lbar}, A'^T and b from shared memory
    const float *ring = p.log + head * (size_t)p.L * p.E;
    float *sA = s_dyn;                        // [c][D]  A'^T
    float *sB = s_dyn + (size_t)p.L * D;      // [c][D]  b
    float *sRaw = s_dyn + (size_t)2 * p.L * D;  // [c][E]  the entries as stored
    // the part of a row the merge reads: whole rows when they hold nothing unused
    // (per-key decay, compact rows), else a | b | Lambda_0 (scalar decay) or a | b
    const int ecopy = (p.a16 || DECAY == DL_DECAY_DIAG) ? p.E : DECAY == DL_DECAY_SCALAR ? p.loff + 4 : p.loff;
    const int nv = ecopy / 4;  // 16-byte vectors per entry
    for (int idx = tid; idx < c * nv; idx += MH_NT) {
        const size_t o = (size_t)(idx / nv) * p.E + 4 * (idx % nv);
        ptx::cp_async16(sRaw + o, ring + o);
    }
    ptx::cp_async_wait_all();
    __syncthreads();
    for (int r = tid; r < D; r += MH_NT) {
        float lb = 0.f;
        if (c > 0 && DECAY == DL_DECAY_DIAG) lb = sRaw[(size_t)(c - 1) * p.E + p.loff + r];
        if (c > 0 && DECAY == DL_DECAY_SCALAR) lb = sRaw[(size_t)(c - 1) * p.E + p.loff];
        s_lb[r] = lb;
        s_e[r] = DECAY == DL_DECAY_NONE ? 1.f : expf(lb);
    }
    __syncthreads();
    for (int idx = tid; idx < c * (D / 4); idx += MH_NT) {
        const int i = idx / (D / 4), r4 = idx % (D / 4);
        const float *ent = sRaw + (size_t)i * p.E;
        float4 a4 = ent_a4(p, ent, r4);
        if (DECAY == DL_DECAY_DIAG) {
            const float4 L4 = *reinterpret_cast<const float4 *>(ent + p.loff + 4 * r4);
            const float4 lb4 = reinterpret_cast<const float4 *>(s_lb)[r4];
            a4.x *= expf(lb4.x - L4.x);
            a4.y *= expf(lb4.y - L4.y);
            a4.z *= expf(lb4.z - L4.z);
            a4.w *= expf(lb4.w - L4.w);
        } else if (DECAY == DL_DECAY_SCALAR) {
            const float g = expf(s_lb[0] - ent[p.loff]);
            a4.x *= g;
            a4.y *= g;
            a4.z *= g;
            a4.w *= g;
        }
        reinterpret_cast<float4 *>(sA + (size_t)i * D)[r4] = a4;
        reinterpret_cast<float4 *>(sB + (size_t)i * D)[r4] = ent_b4(p, ent, r4);
    }
    __syncthreads();

    // 3. the rank-c update of this warp's rows
#pragma unroll
    for (int r4 = 0; r4 < RW / 4; ++r4) {
        const float4 e4 = reinterpret_cast<const float4 *>(s_e + RW * w)[r4];
        const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            float4 &v = S[4 * r4 + y];
            v.x *= ev[y];
            v.y *= ev[y];
            v.z *= ev[y];
            v.w *= ev[y];
        }
    }
    for (int i = 0; i < c; ++i) {
        const float4 b4 = reinterpret_cast<const float4 *>(sB + (size_t)i * D)[lane];
        const float4 *arow = reinterpret_cast<const float4 *>(sA + (size_t)i * D + RW * w);
#pragma unroll
        for (int r4 = 0; r4 < RW / 4; ++r4) {
            const float4 a4 = arow[r4];
            fma4(S[4 * r4 + 0], a4.x, b4);
            fma4(S[4 * r4 + 1], a4.y, b4);
            fma4(S[4 * r4 + 2], a4.z, b4);
            fma4(S[4 * r4 + 3], a4.w, b4);
        }
    }
    float *dst = materialize ? p.dense_out + ((size_t)bi * p.H + h) * (size_t)(D * D) : tile;
#pragma unroll
    for (int r = 0; r < RW; ++r)
        __stcs(reinterpret_cast<float4 *>(dst + (size_t)(RW * w + r) * D) + lane, S[r]);

    // 4. Finalize (merge): the last CTA of this (slot, layer) commits live length 0
    if (!materialize) {
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const int old = atomicAdd(p.arrive + sl, 1);
            if (old == p.H - 1) {
                p.log_len[sl] = 0;
                p.arrive[sl] = 0;
            }
        }
    }
}

}  // namespace dl
