// Warp-per-head decode step for d_k = d_v = 128 (the head shape of every workload
// in the DeltaLog evaluation: 128 x 128 fp32 state per head).
//
// Work unit = one (slot, head), owned by ONE WARP from start to end: the warp
// forms the head's key-side replay coefficients (DeltaLog paper, Section 3.3,
// computed once per slot-head pair), streams the head's 64 KB base state, writes
// o_t and the log entry, and -- as the only owner -- commits the shared log
// metadata.  No CTA-wide barrier exists inside the work loop: the eight warps of
// a CTA work on independent heads, so one head's latencies hide behind the others.
//
// Lane l owns rows 4l..4l+3 for the key-side vectors (q, k, lbar_t, a_i,
// Lambda_i, A'_i) and columns 4l..4l+3 for the value side (v, b_i, o_t, and the
// mat-vec accumulators).  The mat-vecs S^T qt and S^T kt need every row's qt/kt
// in every lane: the owning lanes write the head's row vectors (qt, kt, e^{lbar_t},
// k, lbar_t) to a small per-warp shared-memory area once, and every lane reads
// them as broadcasts, so each lane accumulates its four columns over all 128 rows
// with no cross-lane reduction.  Replay dot products (q^T A'_i, k^T A'_i) are warp
// butterfly sums.
//
// One stream per warp.  Each warp has a ring of NSW shared-memory stages of 8 KB;
// lane 0 keeps NSW copies in flight with cp.async.bulk (TMA bulk copies, mbarrier
// complete_tx), running ahead from one head into the warp's next head.  A head's
// stream is
//     its live log entries, newest first, EPC whole entries per stage,
//     its base state, 16 rows per stage (pass 1: the mat-vecs),
//     its base state again (pass 2), on a merge step under the delta rule,
// so the replay reads entries from shared memory instead of waiting on one load
// after another, and the newest entry -- whose Lambda is lbar -- arrives first.
//
// Merge step (the slot's L-th step): S_t = e^{lbar_t} (.) Sbar + sum_{i<c} A'_i b_i^T
// + k_t b_t^T with A'_i = a_i (.) e^{lbar_t - Lambda_i}.  While replaying, the warp
// also stores A'_i (its rows) and b_i (its columns) of up to TM_ENT entries into its
// share of tensor memory (TMEM, 256 columns x 32 lanes per warp).  Without the delta
// rule b_t = v_t is known from the start, so the new rows are written during pass 1
// itself: the tile is read once and written once.  Under the delta rule b_t needs
// all of pass 1, so the rows are written in pass 2, which re-reads the tile from L2
// (pass-1 copies ask L2 to keep it).  Logs longer than TM_ENT entries (log_cap > 32)
// merge in rounds of MRB entries staged in shared memory instead.
//
// Order of work.  Which heads a CTA takes: with a batch of at most BAL_ROWS slots on a
// decode step that can merge, and one to three heads per warp (where a CTA's merges
// decide its time), every CTA reads the whole batch's slot ids and live
// lengths (all threads at once, one load each) and applies the same rule: the merge
// heads of the launch are dealt round-robin over the CTAs, and each CTA takes a
// contiguous share of the append heads sized so that every CTA's cost (a merge head
// counted as 2 + (L-1)/16 append heads) is about equal.  Otherwise the CTA's heads are
// blockIdx.x + k * gridDim.x.  With more than one head (and at most KMAX), the CTA
// reads its heads' slot ids and live lengths first and puts the merge steps first: a
// merge head costs several append heads, and started early it overlaps their
// streaming instead of ending the launch alone.  When the CTA has few heads, a merge without the delta
// rule is split into 2 or 4 work items, each streaming and rewriting its share of the
// tile's rows (each stages the coefficients in its own TMEM share) and adding its
// partial output into a shared-memory accumulator of the head; the last part to
// arrive adds the token term, writes o_t and commits the head.  Nothing waits for
// another part.  Warps take the items in that order from a shared counter.
//
// The kernel is instantiated per log layout (FMT 0: fp32 rows; FMT 1: compact rows,
// bf16 a_i and, without the delta rule, bf16 b_i), which fixes how many entries a
// stage carries and where each part of an entry sits.  It is launched with
// programmatic stream serialization: a CTA sets up its mbarriers and TMEM while the
// previous kernel in the stream finishes, and reads global memory only after it.
//
// Every wait is bounded (100 ms); a warp whose wait runs out sets DL_EBIT_TIMEOUT,
// stops, and waits (bounded again) for its own copies still in flight before the
// CTA frees its tensor memory and exits.  A test can make that happen on purpose
// (p.stall_ns): the first warp of the first CTA then waits, bounded by stall_ns, on
// a barrier that nothing completes, before it consumes anything of its stream.
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
constexpr int RPB = 4;                      // log entries per load block (merge rounds)
constexpr int MRB = CF / (DK + DV);         // entries per merge round (A' and b in one stage)
constexpr uint64_t WAIT_NS = 100000000ull;  // bound on every wait
constexpr int NB = NSW + 3;                 // mbarriers per warp: stream stages, merge re-stream, stall test
constexpr int TM_ENT = 32;                  // merge entries staged in TMEM per warp
constexpr uint32_t TM_COLS = 512;           // TMEM columns per CTA (all of them)
constexpr uint32_t TM_WCOLS = 256;          // per warp: two warps share each lane quarter
constexpr int AG = 4;                       // merge entries per TMEM load / shared-memory publish
// per-warp scratch: the head's row vectors qt, kt, e^{lbar_t}, k, lbar_t (5 x 128 floats)
// and the A' values of AG entries for the 16 rows of one block
constexpr int WSCR = 5 * DK + AG * CR;
// per-CTA head list: item index, slot id, live length, split combine state of up to
// KMAX heads, and the processing order (a head split in S parts takes S positions)
constexpr int KMAX = 256;
constexpr int MAX_PARTS = 4;                // parts of a split merge head
constexpr int NPA = 8;                      // split heads in flight per CTA (accumulators)
// balanced schedule: the whole batch's slot ids and live lengths, and a bitmap of its
// merging rows with per-word prefix counts
constexpr int BAL_ROWS = 512;
constexpr int LMAX = 64;                    // largest log capacity (bins of the longest-first order)
constexpr int BAL_WORDS = BAL_ROWS / 32;
constexpr size_t SMEM = (size_t)NW * NSW * CB + (size_t)NW * WSCR * 4 + (size_t)NW * NB * 8 + 32 +
                        (size_t)KMAX * (4 + 4 + 4 + 4) + (size_t)2 * KMAX * 2 + (size_t)NPA * DV * 4 +
                        (size_t)BAL_ROWS * (4 + 1) + (size_t)BAL_WORDS * (4 + 4) + (size_t)(LMAX + 2) * 4;
static_assert(KMAX + (MAX_PARTS - 1) * NPA <= 2 * KMAX, "the order holds every head and every extra part");
static_assert(SMEM <= 232448, "a CTA may use at most 227 KB of shared memory");
static_assert(NSW == 3, "the round-wise merge uses stages 0-1 for the tile and stage 2 as scratch");
static_assert(TM_ENT * 8 <= (int)TM_WCOLS, "A'_i and b_i take 8 columns per entry");
constexpr unsigned FULL = 0xffffffffu;

// Log entry layout (FMT 0: fp32 [a | b | Lambda]; FMT 1: compact, a bf16, b bf16 without
// the delta rule, Lambda fp32 x d_k / x 4 / absent) and how entries travel through a
// stage.  Whole ring rows are copied when they hold nothing unused (compact rows, or
// per-key decay); otherwise each entry's [a | b | Lambda_0 and 3 pad floats] (scalar
// decay) or [a | b] (no decay) is copied.  Up to EPC entries fill one stage.
template <int DECAY, int FMT, bool DELTA>
struct LogCopy {
    static constexpr bool A16 = FMT == 1;
    static constexpr bool B16 = FMT == 1 && !DELTA;
    static constexpr int B_OFF = A16 ? DK / 2 : DK;            // b_i in floats from the row start
    static constexpr int L_OFF = B_OFF + (B16 ? DV / 2 : DV);   // Lambda_i
    static constexpr int E_F = FMT == 1 ? L_OFF + (DECAY == DL_DECAY_DIAG ? DK : DECAY == DL_DECAY_SCALAR ? 4 : 0)
                                        : 2 * DK + DV;          // ring row in floats
    static constexpr bool WHOLE = FMT == 1 || DECAY == DL_DECAY_DIAG;
    static constexpr uint32_t ESB = WHOLE ? E_F * 4 : (L_OFF + (DECAY == DL_DECAY_SCALAR ? 4 : 0)) * 4;
    static constexpr int ESF = ESB / 4;
    static constexpr int EPC = CB / ESB < 8 ? CB / ESB : 8;     // capped: the replay unrolls a stage
};

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

enum MergeKind : int {
    MK_APPEND = 0,  // append step: o_t from base + log, entry c appended
    MK_FUSED = 1,   // merge without the delta rule: new rows written during pass 1
    MK_PASS2 = 2,   // merge under the delta rule: new rows written in pass 2
    MK_ROUNDS = 3   // merge of more than TM_ENT entries: rounds staged in shared memory
};

// One head as the warp sees it.
struct Head {
    int it;        // work item (batch row * H + head), n_items when past the end
    int s;         // slot id
    int ok;        // slot id in range (the head is processed unless st is set later)
    int c;         // live entries
    int st;        // 0, or the error bit that makes the head skipped
    int mk;        // MergeKind
    int nl;        // log chunks in its stream
    int n;         // stream positions: nl + NCH (+ NCH for MK_PASS2); 0 when skipped
    int part;      // 0: the whole head; 1..np: rows (part-1)*128/np .. part*128/np - 1 of a split merge
    int np;        // parts of a split merge head
    int k;         // place in the CTA's head list (when there is one)
    size_t head;   // (slot, layer, head) index
};

// a_i[4l .. 4l + 3] or b_i[4l .. 4l + 3] of an entry (shared or global memory)
template <bool HALF>
__device__ __forceinline__ float4 seg4(const float *seg, int lane) {
    if (HALF) {
        const uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(seg) + 4 * lane);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
        return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
    }
    return reinterpret_cast<const float4 *>(seg)[lane];
}
// the values stored narrow are bf16 inputs (k_t; v_t without the delta rule): exact
template <bool HALF>
__device__ __forceinline__ void put_seg4(float *seg, int lane, float4 v) {
    if (HALF) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&lo);
        u.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(reinterpret_cast<__nv_bfloat16 *>(seg) + 4 * lane) = u;
    } else {
        reinterpret_cast<float4 *>(seg)[lane] = v;
    }
}

template <int DECAY, bool DELTA, typename IT, int FMT>
__global__ void __launch_bounds__(NTHREADS, 1) warp_head_kernel(const KParams p)
{
    using LC = LogCopy<DECAY, FMT, DELTA>;
    constexpr uint32_t ESB = LC::ESB;
    constexpr int ESF = LC::ESF, EPC = LC::EPC;
    constexpr int BO = LC::B_OFF, LO = LC::L_OFF;

    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float *st = reinterpret_cast<float *>(smem) + (size_t)w * NSW * CF;
    float *rv = reinterpret_cast<float *>(smem + (size_t)NW * NSW * CB) + (size_t)w * WSCR;
    float *rv_qt = rv, *rv_kt = rv + DK, *rv_e = rv + 2 * DK, *rv_k = rv + 3 * DK, *rv_l = rv + 4 * DK;
    float *ag = rv + 5 * DK;
    unsigned char *bars = smem + (size_t)NW * NSW * CB + (size_t)NW * WSCR * 4;
    uint64_t *fb = reinterpret_cast<uint64_t *>(bars) + w * NB;
    uint64_t *pb = fb + NSW;  // round-wise merge: tile re-stream through stages 0 and 1
    uint64_t *stall_bar = fb + NSW + 2;  // nothing ever arrives on it (timeout test)
    int *next_k = reinterpret_cast<int *>(bars + (size_t)NW * NB * 8);
    uint32_t *tm_slot = reinterpret_cast<uint32_t *>(next_k + 1);
    int *cnt = next_k + 2;  // merge positions, next merge position, next other position, extra parts,
                            // accumulators taken, merging rows of the batch (balanced schedule)
    int *pre_it = next_k + 8;    // item index (batch row * H + head) of the CTA's k-th head
    int *pre_slot = pre_it + KMAX;
    int *pre_len = pre_slot + KMAX;
    int *comb = pre_len + KMAX;  // split merge heads: (accumulator + 1) << 8 | parts arrived
    uint16_t *order = reinterpret_cast<uint16_t *>(comb + KMAX);  // k | part << 10 | log2(parts) << 13
    float *pacc = reinterpret_cast<float *>(order + 2 * KMAX);  // NPA x DV partial outputs
    int *row_slot = reinterpret_cast<int *>(pacc + NPA * DV);   // balanced schedule: per batch row
    unsigned *bmap = reinterpret_cast<unsigned *>(row_slot + BAL_ROWS);  // merging rows
    int *wpre = reinterpret_cast<int *>(bmap + BAL_WORDS);      // set bits before each word
    // append heads per live length, then the next position of each (longest first)
    int *lbin = wpre + BAL_WORDS;
    uint8_t *row_len = reinterpret_cast<uint8_t *>(lbin + LMAX + 2);

    // merges with live entries need tensor memory (auto-merge decode steps only)
    const bool use_tm = p.auto_merge && !p.eager && p.log != nullptr;
    if (lane == 0) {
        for (int s = 0; s < NB; ++s) ptx::mbar_init(&fb[s], 1);
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 0) {
        *next_k = NW;  // warp w starts with the CTA's w-th head
        cnt[0] = cnt[1] = cnt[2] = cnt[3] = cnt[4] = 0;
    }
    for (int i = threadIdx.x; i < NPA * DV; i += NTHREADS) pacc[i] = 0.f;
    for (int i = threadIdx.x; i < BAL_WORDS; i += NTHREADS) bmap[i] = 0u;
    for (int i = threadIdx.x; i < LMAX + 2; i += NTHREADS) lbin[i] = 0;
    if (use_tm && w == 0) {
        ptx::tmem_alloc(tm_slot, TM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tmem_fence_before_sync();
    __syncthreads();
    ptx::tmem_fence_after_sync();
    // Only on-chip state was touched so far.  With programmatic dependent launch this
    // CTA may have started while the previous kernel in the stream was finishing:
    // global memory is read only after that kernel has completed.  The next launch
    // may then begin (its CTAs take an SM only when this one leaves it).
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    // this warp's TMEM: lanes of its quarter, columns of its half
    const uint32_t tm = use_tm ? *tm_slot + ((uint32_t)(32 * (w & 3)) << 16) + TM_WCOLS * (uint32_t)(w >> 2)
                               : 0u;

    const int n_items = p.batch * p.H;
    const int G = gridDim.x, bx = blockIdx.x;
    auto merges = [&](int s, int c) {
        return s >= 0 && s < p.n_slots && (p.eager || (p.auto_merge && (c >= p.L - 1 || p.merge_every)));
    };
    int kc = bx < n_items ? (n_items - 1 - bx) / G + 1 : 0;  // heads of this CTA (natural order)
    // Balanced schedule (see the header): a decode step that can merge, with at most
    // BAL_ROWS rows and one to three heads per warp on average.  With fewer, a CTA's
    // time is its slowest warp, and the natural assignment already gives each CTA at
    // most one item per warp.  With more, the merges of a CTA are a small part of its
    // work and the natural, strided assignment streams faster: at any moment the
    // whole GPU reads a window of consecutive heads, where contiguous per-CTA ranges
    // spread the reads over the whole state (measured on B200: KDA, 55 heads per CTA,
    // 0.80 against 0.86 of the copy rate).
    bool bal = !p.eager && p.auto_merge && p.log_len && p.batch <= BAL_ROWS &&
               (long long)n_items >= (long long)G * NW && (long long)n_items < (long long)G * 3 * NW;
    if (bal) {
        // every batch row's slot id and live length; merging rows set their bit
        constexpr int RPT = BAL_ROWS / NTHREADS;
        int sv[RPT];
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int b = threadIdx.x + j * NTHREADS;
            sv[j] = b < p.batch ? p.slots[b] : -1;
        }
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int b = threadIdx.x + j * NTHREADS;
            if (b >= p.batch) continue;
            const bool ok = sv[j] >= 0 && sv[j] < p.n_slots;
            const int c = ok ? p.log_len[(size_t)sv[j] * p.n_layers + p.layer] : 0;
            row_slot[b] = sv[j];
            row_len[b] = (uint8_t)(c < 0 ? 255 : c > 254 ? 254 : c);  // out of [0, L]: flagged at the head
            if (ok && merges(sv[j], c)) atomicOr(&bmap[b >> 5], 1u << (b & 31));
        }
        __syncthreads();
        const int nwords = (p.batch + 31) >> 5;
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int i = 0; i < nwords; ++i) {
                wpre[i] = acc;
                acc += __popc(bmap[i]);
            }
            cnt[5] = acc;  // merging rows of the batch
        }
        __syncthreads();
        // Integer costs in 1/16 of an append head (n_items <= G * KMAX / 4, so every
        // quantity below fits 32 bits except the product in A()).  Nothing here loops
        // over CTAs: this runs at the start of every launch.
        const int NMH = cnt[5] * p.H, NA = n_items - NMH;
        const int Wm = 32 + (p.L - 1);  // a merge head costs 2 + (L-1)/16 append heads
        const int q = NMH / G, r = NMH % G;
        const int target = (16 * NA + Wm * NMH) / G;
        const int cap_lo = target > Wm * (q + 1) ? target - Wm * (q + 1) : 0;  // CTAs with q+1 merges
        const int cap_hi = target > Wm * q ? target - Wm * q : 0;              // CTAs with q merges
        auto P = [&](int x) -> long long {
            return (long long)(x < r ? x : r) * cap_lo + (long long)(x > r ? x - r : 0) * cap_hi;
        };
        const long long PG = P(G);
        auto A = [&](int x) -> int { return PG > 0 ? (int)((long long)NA * P(x) / PG) : (int)((long long)NA * x / G); };
        // the same decision in every CTA: fall back unless every CTA's share fits the list
        // (a CTA takes at most q + 1 merge heads and NA * cap / PG + 1 append heads)
        const int cap_max = cap_lo > cap_hi ? cap_lo : cap_hi;
        const long long kbound = q + 1 + (PG > 0 ? (long long)NA * cap_max / PG : (long long)NA / G) + 1;
        if (kbound > KMAX) {
            bal = false;
        } else {
            const int km = q + (bx < r ? 1 : 0);
            const int a0 = A(bx);
            kc = km + (A(bx + 1) - a0);
            // row of the j-th merging / non-merging batch row
            auto select = [&](int j, bool set) -> int {
                int wd = 0;
                auto before = [&](int i) -> int { return set ? wpre[i] : 32 * i - wpre[i]; };
                while (wd + 1 < nwords && before(wd + 1) <= j) ++wd;
                unsigned m = set ? bmap[wd] : ~bmap[wd];
                for (int rem = j - before(wd); rem > 0; --rem) m &= m - 1;
                return 32 * wd + __ffs(m) - 1;
            };
            for (int k = threadIdx.x; k < kc; k += NTHREADS) {
                const int u = k < km ? bx + k * G : a0 + (k - km);  // merge / append head u of the launch
                const int row = select(u / p.H, k < km);
                pre_it[k] = row * p.H + u % p.H;
                pre_slot[k] = row_slot[row];
                pre_len[k] = row_len[row] == 255 ? -1 : row_len[row];
            }
        }
    }
    // the head list is built when there is an order to choose (more heads than warps),
    // and always for the balanced schedule; with at most one head per warp each warp
    // reads its own head's metadata, which measured faster than building the list
    // (GLA B = 64: 0.66 against 0.74 of the copy rate with merges synchronised)
    const bool pre = bal || (kc > NW && kc <= KMAX);
    // Merges written during pass 1 (no delta rule, at most TM_ENT entries) are split
    // when the CTA has few heads: a merge head costs several append heads (its
    // write-back is a chain of c-term updates run by one warp), so with fewer than
    // three heads per warp it would outlast the rest of the CTA's work; with more,
    // the other heads hide it and a split only adds the parts' log reads.  Parts:
    // with fewer heads than warps, as many as the idle warps allow (2 or 4); else 2,
    // or 4 for logs of 16 entries or more.
    const bool split_ok = kc < 3 * NW;
    auto parts_of = [&](int s, int c) -> int {
        if (!(split_ok && !DELTA && !p.eager && p.want_out && merges(s, c) && c >= 0 && c <= TM_ENT)) return 1;
        if (kc < NW) return NW - kc >= 3 ? 4 : NW - kc >= 1 ? 2 : 1;
        return c >= 16 ? 4 : 2;
    };
    if (pre) {
        if (!bal) {
            for (int k = threadIdx.x; k < kc; k += NTHREADS) {
                const int it = bx + k * G;
                const int s = p.slots[it / p.H];
                pre_it[k] = it;
                pre_slot[k] = s;
                pre_len[k] = (s >= 0 && s < p.n_slots && p.log_len) ? p.log_len[(size_t)s * p.n_layers + p.layer]
                                                                     : 0;
            }
        }
        __syncthreads();
        for (int k = threadIdx.x; k < kc; k += NTHREADS) {
            const int s = pre_slot[k], c = pre_len[k];
            int np = parts_of(s, c);
            int cm = 0;
            if (np > 1) {  // a split head needs one of the NPA accumulators
                const int a = atomicAdd(&cnt[4], 1);
                if (a < NPA) cm = (a + 1) << 8;
                else np = 1;
            }
            comb[k] = cm;
            if (merges(s, c)) atomicAdd(&cnt[0], np);
            else atomicAdd(&lbin[c < 0 || c > LMAX ? 0 : c], 1);
            if (np > 1) atomicAdd(&cnt[3], np - 1);
        }
        __syncthreads();
        // Append heads in order of decreasing live length (longest first): a head with
        // c live entries streams and replays c log entries besides its tile, so the
        // short ones end the order and the warps finish closer together.  lbin[c]
        // becomes the first append position of live length c.
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int cc = LMAX; cc >= 0; --cc) {
                const int n = lbin[cc];
                lbin[cc] = acc;
                acc += n;
            }
        }
        __syncthreads();
        const int nm = cnt[0];
        // With many heads per warp (8 or more; no splits then, one position per head)
        // and merges written during pass 1, the merge heads are spread evenly over all
        // but the last NW positions: started all at once, their write-back (ALU work)
        // would leave the SM with few streaming warps at the start of the launch
        // (RetNet B = 1024: 0.905 -> 0.949 of the copy rate).  Otherwise they go first:
        // with fewer heads the launch's tail must not end on a merge, and delta-rule
        // merges, which re-read their tile from L2 in pass 2, measured slower spread
        // (KDA: 0.86 -> 0.73).
        const int span = kc - NW;
        const bool spread = !DELTA && kc >= 8 * NW && nm > 0 && span >= nm;
        auto merge_pos = [&](int i) { return spread ? (int)((long long)i * span / nm) : i; };
        for (int k = threadIdx.x; k < kc; k += NTHREADS) {
            const int s = pre_slot[k], c = pre_len[k];
            if (comb[k] != 0) {
                const int np = parts_of(s, c), lg = np == 4 ? 2 : 1;
                const int pos = atomicAdd(&cnt[1], np);  // the parts next to each other
                for (int j = 0; j < np; ++j) order[pos + j] = (uint16_t)(k | ((j + 1) << 10) | (lg << 13));
            } else if (merges(s, c)) {
                order[merge_pos(atomicAdd(&cnt[1], 1))] = (uint16_t)k;
            } else {
                const int a = atomicAdd(&lbin[c < 0 || c > LMAX ? 0 : c], 1);  // longest first
                int pos = a;  // the a-th position no merge head takes
                if (spread) {
                    for (int i = 0; i < nm && merge_pos(i) <= pos; ++i) ++pos;
                } else {
                    pos += nm;
                }
                order[pos] = (uint16_t)k;
            }
        }
        __syncthreads();
    }
    const int npos = pre ? kc + cnt[3] : kc;  // work items of this CTA
    // work item at a position of the order: the head's item index, its part and its
    // place k in the CTA's list (pinfo = part | parts << 4 | k << 8; part 0: whole head)
    auto item_at = [&](int pos, int &pinfo) -> int {
        pinfo = 0;
        if (pos >= npos) return n_items;
        if (!pre) return bx + pos * G;
        const int o = order[pos];
        const int part = (o >> 10) & 7, k = o & 1023;
        pinfo = k << 8;
        if (part) pinfo |= part | ((1 << (o >> 13)) << 4);
        return pre_it[k];
    };
    // warps take the next position from a shared counter as they finish, so a warp
    // held up by a merge head takes fewer heads
    auto grab = [&](int &pinfo) -> int {
        int pos = 0;
        if (lane == 0) pos = atomicAdd(next_k, 1);
        return item_at(__shfl_sync(FULL, pos, 0), pinfo);
    };
    const int E = p.E;
    const uint64_t pol_stream = ptx::policy_evict_first();
    const uint64_t pol_keep = ptx::policy_evict_last();

    // -- head metadata: slot id first (it locates the tile and the log), live
    //    length after (it sizes the log part of the stream and decides the merge)
    auto slot_of = [&](int it, int pinfo) -> int {
        if (it >= n_items) return -1;
        return pre ? pre_slot[pinfo >> 8] : p.slots[it / p.H];
    };
    auto len_of = [&](const Head &hd) -> int {
        if (!hd.ok) return 0;
        if (pre) return pre_len[hd.k];
        return p.log_len ? p.log_len[(size_t)hd.s * p.n_layers + p.layer] : 0;
    };
    auto resolve_slot = [&](Head &hd, int it, int s, int pinfo) {
        hd.it = it;
        hd.part = pinfo & 15;
        hd.np = (pinfo >> 4) & 15;
        hd.k = pinfo >> 8;
        hd.s = s;
        hd.ok = 0;
        hd.c = 0;
        hd.st = 0;
        hd.mk = MK_APPEND;
        hd.nl = 0;
        hd.n = 0;
        hd.head = 0;
        if (it >= n_items) return;
        if (s < 0 || s >= p.n_slots) { hd.st = DL_EBIT_SLOT_RANGE; return; }
        hd.head = ((size_t)s * p.n_layers + p.layer) * p.H + (it % p.H);
        hd.ok = 1;
    };
    auto resolve_len = [&](Head &hd, int c) {
        if (!hd.ok) return;
        hd.c = c;
        if (p.eager) {
            if (c != 0) hd.st = DL_EBIT_LIVE_LOG;
        } else if (c < 0 || c > p.L) {
            hd.st = DL_EBIT_LOG_LEN;
        } else if (!(p.auto_merge && (c >= p.L - 1 || p.merge_every)) && c >= p.L) {
            hd.st = DL_EBIT_LOG_FULL;
        }
        if (hd.st) return;
        const bool merge = p.eager || (p.auto_merge && (c >= p.L - 1 || p.merge_every));
        hd.mk = !merge ? MK_APPEND : c > TM_ENT ? MK_ROUNDS : DELTA ? MK_PASS2 : MK_FUSED;
        hd.nl = (c + EPC - 1) / EPC;
        hd.n = hd.nl + (hd.part ? NCH / hd.np : NCH) + (hd.mk == MK_PASS2 ? NCH : 0);
    };
    // L2 warm-up of a head's token rows (they depend on the work item only)
    auto warm_token = [&](int it) {
        if (lane != 0 || it >= n_items) return;
        const int bi = it / p.H, h = it % p.H, gk = h / (p.H / p.Hk);
        ptx::prefetch_l2(static_cast<const IT *>(p.q) + ((size_t)bi * p.Hk + gk) * DK, DK * sizeof(IT));
        ptx::prefetch_l2(static_cast<const IT *>(p.k) + ((size_t)bi * p.Hk + gk) * DK, DK * sizeof(IT));
        ptx::prefetch_l2(static_cast<const IT *>(p.v) + ((size_t)bi * p.H + h) * DV, DV * sizeof(IT));
        if (DECAY == DL_DECAY_DIAG && !p.lam_const)
            ptx::prefetch_l2(p.lam + ((size_t)bi * p.H + h) * DK, DK * 4);
    };

    // -- the warp's stream: positions [base, base + cur.n) belong to cur, then up to
    //    nxt.n positions of nxt (issued once nxt's live length is known)
    int gc = 0, gi = 0, base = 0;  // consumed / issued stream positions
    bool abort = false;
    uint32_t pph = 0u;             // round-wise merge re-stream barrier phases (bit b: pb[b])
    uint32_t pb_pend = 0u;         // round-wise merge re-stream copies in flight (bit b)
    Head cur, nxt;
    nxt.ok = 0;
    nxt.n = 0;
    int pinfo0 = 0, pinfo_nxt = 0;  // part info of the current and the next item
    const int it0 = item_at(w, pinfo0);
    warm_token(it0);
    resolve_slot(cur, it0, slot_of(it0, pinfo0), pinfo0);
    int it_nxt = grab(pinfo_nxt);         // the warp's next head, and its slot id, one head early
    int s_nxt = slot_of(it_nxt, pinfo_nxt);
    bool nxt_res = false;                // nxt's live length known
    int c_nxt = 0;

    // position x of head hd into stage gi % NSW (lane 0)
    auto issue_pos = [&](const Head &hd, int x) {
        const int sg = gi % NSW;
        uint64_t *bar = &fb[sg];
        float *dst = st + (size_t)sg * CF;
        if (x < hd.nl) {
            const int hi = hd.c - EPC * x, lo = hi - EPC > 0 ? hi - EPC : 0;
            const float *src = p.log + hd.head * (size_t)p.L * E;
            ptx::mbar_arrive_expect_tx(bar, (uint32_t)(hi - lo) * ESB);
            if (LC::WHOLE) {
                ptx::bulk_g2s(dst, src + (size_t)lo * E, (uint32_t)(hi - lo) * ESB, bar, pol_stream);
            } else {
                for (int i = lo; i < hi; ++i)
                    ptx::bulk_g2s(dst + (size_t)(i - lo) * ESF, src + (size_t)i * E, ESB, bar, pol_stream);
            }
        } else {
            const int y = x - hd.nl + (hd.part ? (hd.part - 1) * (NCH / hd.np) : 0);  // a part's first chunk
            const bool keep = y < NCH && hd.mk == MK_ROUNDS;
            ptx::mbar_arrive_expect_tx(bar, CB);
            ptx::bulk_g2s(dst, p.state + hd.head * (size_t)(DK * DV) + (size_t)(y & (NCH - 1)) * CF, CB, bar,
                          keep ? pol_keep : pol_stream);
        }
    };
    auto issue_upto = [&](int limit) {
        while (gi < limit) {
            if (gi < base + cur.n) {
                if (lane == 0) issue_pos(cur, gi - base);
                ++gi;
                continue;
            }
            // a round-wise merge needs its stages as scratch after pass 1: no look-ahead
            if ((cur.mk == MK_ROUNDS && cur.st == 0) || !nxt.ok) break;
            if (!nxt_res) {
                resolve_len(nxt, c_nxt);
                nxt_res = true;
            }
            const int rel = gi - base - cur.n;
            if (rel >= nxt.n) break;
            if (lane == 0) issue_pos(nxt, rel);
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

    // The first head has no head before it to hide its prologue.  Its dependent
    // loads (slot id, then live length) go out before any of its stream does.
    resolve_len(cur, len_of(cur));
    issue_upto(NSW);

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
        if (p.stall_ns && bx == 0 && w == 0 && gc == 0) {
            // timeout test: a wait that runs out, with the warp's first copies in flight
            const bool ok = ptx::mbar_wait_bounded(stall_bar, 0u, p.stall_ns);
            if (!__all_sync(FULL, ok)) { abort = true; break; }
        }
        // the next head: slot id read one head ago; its live length is loaded now
        // and used when the stream reaches it
        resolve_slot(nxt, it_nxt, s_nxt, pinfo_nxt);
        nxt_res = false;
        c_nxt = len_of(nxt);
        if (nxt.ok) warm_token(nxt.it);
        if (cur.st && lane == 0) atomicOr(p.err, cur.st);

        if (cur.st == 0) {
            const int c = cur.c, mk = cur.mk;
            const int bi = cur.it / p.H, h = cur.it % p.H;
            const size_t row = (size_t)bi * p.H + h;
            const size_t sl = (size_t)cur.s * p.n_layers + p.layer;
            float *tile = p.state + cur.head * (size_t)(DK * DV);
            float *ring = p.log ? p.log + cur.head * (size_t)p.L * E : nullptr;
            const int gk = h / (p.H / p.Hk);
            const bool stage_tm = use_tm && c > 0 && (mk == MK_FUSED || mk == MK_PASS2);

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
            } else if (DECAY == DL_DECAY_SCALAR) {
                const float ls = __ldg(p.lam + (p.lam_const ? (size_t)h : row));
#pragma unroll
                for (int x = 0; x < 4; ++x) lam[x] = ls;
            }
            // lbar = Lambda of the newest entry, the last row of the first log chunk
            if (c > 0) {
                if (!wait_chunk()) { abort = true; break; }
                const int lo0 = c - EPC > 0 ? c - EPC : 0;
                const float *ent = st + (size_t)(gc % NSW) * CF + (size_t)(c - 1 - lo0) * ESF + LO;
                if (DECAY == DL_DECAY_DIAG) {
                    const float4 p4 = reinterpret_cast<const float4 *>(ent)[lane];
                    lp[0] = p4.x; lp[1] = p4.y; lp[2] = p4.z; lp[3] = p4.w;
                } else if (DECAY == DL_DECAY_SCALAR) {
                    const float ps = ent[0];
#pragma unroll
                    for (int x = 0; x < 4; ++x) lp[x] = ps;
                }
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
            // row vectors for the row blocks' broadcasts
            reinterpret_cast<float4 *>(rv_qt)[lane] = make_float4(qt[0], qt[1], qt[2], qt[3]);
            if (DELTA) reinterpret_cast<float4 *>(rv_kt)[lane] = make_float4(kt[0], kt[1], kt[2], kt[3]);
            reinterpret_cast<float4 *>(rv_e)[lane] = make_float4(e_own[0], e_own[1], e_own[2], e_own[3]);
            reinterpret_cast<float4 *>(rv_k)[lane] = make_float4(k_own[0], k_own[1], k_own[2], k_own[3]);
            reinterpret_cast<float4 *>(rv_l)[lane] = make_float4(ell[0], ell[1], ell[2], ell[3]);
            __syncwarp();

            // -- ReplayPrep + value replay over the log chunks (newest first):
            //    Y += (q^T A'_i) b_i, (k^T A'_i) b_i; a merge also stages A'_i, b_i in TMEM
            float4 Yq = make_float4(0.f, 0.f, 0.f, 0.f), Yk = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int x = 0; x < cur.nl; ++x) {
                if (x > 0 && !wait_chunk()) { abort = true; break; }
                const float *sb = st + (size_t)(gc % NSW) * CF;
                const int hi = c - EPC * x, lo = hi - EPC > 0 ? hi - EPC : 0;
                float pq[EPC], pk[EPC];
#pragma unroll
                for (int e = 0; e < EPC; ++e) {
                    pq[e] = 0.f;
                    pk[e] = 0.f;
                    if (lo + e < hi) {
                        const float *ent = sb + (size_t)e * ESF;
                        const float4 a4 = seg4<LC::A16>(ent, lane);
                        float Lv[4] = {0.f, 0.f, 0.f, 0.f};
                        if (DECAY == DL_DECAY_DIAG) {
                            const float4 L4 = reinterpret_cast<const float4 *>(ent + LO)[lane];
                            Lv[0] = L4.x; Lv[1] = L4.y; Lv[2] = L4.z; Lv[3] = L4.w;
                        } else if (DECAY == DL_DECAY_SCALAR) {
                            const float Ls = ent[LO];
#pragma unroll
                            for (int y = 0; y < 4; ++y) Lv[y] = Ls;
                        }
                        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
                        float wq[4];
#pragma unroll
                        for (int y = 0; y < 4; ++y) {
                            const float g = DECAY == DL_DECAY_NONE ? 1.f : expf(ell[y] - Lv[y]);
                            wq[y] = av[y] * g;
                            pq[e] = fmaf(wq[y], q_own[y], pq[e]);
                            if (DELTA) {
                                const float wk = (p.undecayed && DECAY != DL_DECAY_NONE)
                                                     ? av[y] * expf(lp[y] - Lv[y]) : wq[y];
                                pk[e] = fmaf(wk, k_own[y], pk[e]);
                            }
                        }
                        if (stage_tm) {
                            const float4 b4 = seg4<LC::B16>(ent + BO, lane);
                            const float tv[8] = {wq[0], wq[1], wq[2], wq[3], b4.x, b4.y, b4.z, b4.w};
                            ptx::tmem_st8(tm + 8u * (uint32_t)(lo + e), tv);
                        }
                    }
                }
                // butterfly sums of the chunk's entries, level by level
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) {
                        pq[e] += __shfl_xor_sync(FULL, pq[e], o);
                        if (DELTA) pk[e] += __shfl_xor_sync(FULL, pk[e], o);
                    }
                }
#pragma unroll
                for (int e = 0; e < EPC; ++e) {
                    if (lo + e < hi) {
                        const float4 b4 = seg4<LC::B16>(sb + (size_t)e * ESF + BO, lane);
                        fma4(Yq, pq[e], b4);
                        if (DELTA) fma4(Yk, pk[e], b4);
                    }
                }
                release();
            }
            if (abort) break;
            if (stage_tm) ptx::tmem_wait_st();
            if (cur.part > 1) Yq = make_float4(0.f, 0.f, 0.f, 0.f);  // counted once, by the first part

            // new rows of one 16-row block of the merged state from its Sbar rows in
            // shared memory: e^{lbar_t} Sbar + sum_i A'_i b_i^T + k b_t^T, i ascending.
            // A'_i rows of the block are published AG entries at a time by the block's
            // four owner lanes and read by every lane as broadcasts.
            // (token: add k b_t^T; streaming: evict-first stores, else plain stores that
            //  stay in L2 for pass 2 of a delta-rule merge)
            auto write_rows = [&](const float *sb, int cx, const float4 &bt4, bool token, bool streaming) {
                float4 acc[CR];
#pragma unroll
                for (int r4 = 0; r4 < CR / 4; ++r4) {
                    const float4 e4 = reinterpret_cast<const float4 *>(rv_e + cx * CR)[r4];
                    const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const float4 S = reinterpret_cast<const float4 *>(sb + (4 * r4 + y) * DV)[lane];
                        acc[4 * r4 + y] = make_float4(S.x * ev[y], S.y * ev[y], S.z * ev[y], S.w * ev[y]);
                    }
                }
                const int nj = stage_tm ? c : 0;  // TMEM is read only where it was written
                for (int j0 = 0; j0 < nj; j0 += AG) {
                    float tv[8 * AG];
                    ptx::tmem_ld32(tm + 8u * (uint32_t)j0, tv);
                    if ((lane >> 2) == cx) {
#pragma unroll
                        for (int g = 0; g < AG; ++g)
                            reinterpret_cast<float4 *>(ag + g * CR)[lane & 3] =
                                make_float4(tv[8 * g], tv[8 * g + 1], tv[8 * g + 2], tv[8 * g + 3]);
                    }
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < AG; ++g) {
                        if (j0 + g < nj) {
                            const float4 b4 = make_float4(tv[8 * g + 4], tv[8 * g + 5], tv[8 * g + 6], tv[8 * g + 7]);
#pragma unroll
                            for (int r4 = 0; r4 < CR / 4; ++r4) {
                                const float4 a4 = reinterpret_cast<const float4 *>(ag + g * CR)[r4];
                                fma4(acc[4 * r4 + 0], a4.x, b4);
                                fma4(acc[4 * r4 + 1], a4.y, b4);
                                fma4(acc[4 * r4 + 2], a4.z, b4);
                                fma4(acc[4 * r4 + 3], a4.w, b4);
                            }
                        }
                    }
                    __syncwarp();
                }
#pragma unroll
                for (int r4 = 0; r4 < CR / 4; ++r4) {
                    const float4 k4 = reinterpret_cast<const float4 *>(rv_k + cx * CR)[r4];
                    const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const int rr = 4 * r4 + y;
                        if (token) fma4(acc[rr], kv[y], bt4);
                        float4 *dst = reinterpret_cast<float4 *>(tile + (size_t)(cx * CR + rr) * DV) + lane;
                        if (streaming) __stcs(dst, acc[rr]);
                        else *dst = acc[rr];
                    }
                }
            };

            // -- AppendDecode pass 1: y_q = Sbar^T qt, y_k = Sbar^T kt (columns 4l..4l+3);
            //    without the delta rule a merge writes its new rows here as well
            const float4 v4 = make_float4(v_own[0], v_own[1], v_own[2], v_own[3]);
            const int cx0 = cur.part ? (cur.part - 1) * (NCH / cur.np) : 0;
            const int cx1 = cur.part ? cx0 + NCH / cur.np : NCH;
            for (int cx = cx0; cx < cx1; ++cx) {
                if (!wait_chunk()) { abort = true; break; }
                const float *sb = st + (size_t)(gc % NSW) * CF;
#pragma unroll
                for (int r4 = 0; r4 < CR / 4; ++r4) {
                    const float4 q4 = reinterpret_cast<const float4 *>(rv_qt + cx * CR)[r4];
                    const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
                    float kv[4] = {0.f, 0.f, 0.f, 0.f};
                    if (DELTA) {
                        const float4 k4 = reinterpret_cast<const float4 *>(rv_kt + cx * CR)[r4];
                        kv[0] = k4.x; kv[1] = k4.y; kv[2] = k4.z; kv[3] = k4.w;
                    }
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const float4 S = reinterpret_cast<const float4 *>(sb + (4 * r4 + y) * DV)[lane];
                        fma4(Yq, qv[y], S);
                        if (DELTA) fma4(Yk, kv[y], S);
                    }
                }
                if (!DELTA && mk == MK_FUSED) {
                    write_rows(sb, cx, v4, true, true);
                } else if (DELTA && mk == MK_PASS2) {
                    // e^{lbar_t} Sbar + sum_i A'_i b_i^T now, while the stream is DRAM-bound;
                    // the token term needs b_t, so pass 2 adds it.  Pass 2's bulk copies
                    // re-read these rows (issued at least NCH - NSW stages later): order
                    // the writes before them.
                    write_rows(sb, cx, v4, false, false);
                    ptx::fence_proxy_async_global();
                }
                release();
            }
            if (abort) break;

            finish_commit();

            // -- b_t, o_t, and the append (entry c)
            const float yq[4] = {Yq.x, Yq.y, Yq.z, Yq.w}, yk[4] = {Yk.x, Yk.y, Yk.z, Yk.w};
            float bt[4], o[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                bt[x] = DELTA ? beta * (v_own[x] - yk[x]) : v_own[x];
                o[x] = fmaf(bt[x], kq, yq[x]);
            }
            const float4 bt4 = make_float4(bt[0], bt[1], bt[2], bt[3]);
            bool commits = true;  // this work item finalizes the head
            if (cur.part) {
                // Split merge: every part adds its partial (its rows' share of
                // Sbar^T qt; the first part also the replay) into the head's
                // shared-memory accumulator and counts itself in; the last to arrive
                // adds the token term, writes o_t and commits the head.
                int *cm = comb + cur.k;
                // the accumulator index (high bits) is fixed since the head list was built
                float *acc = pacc + (size_t)((*reinterpret_cast<volatile int *>(cm) >> 8) - 1) * DV + 4 * lane;
                atomicAdd(acc + 0, Yq.x);
                atomicAdd(acc + 1, Yq.y);
                atomicAdd(acc + 2, Yq.z);
                atomicAdd(acc + 3, Yq.w);
                __threadfence_block();
                __syncwarp();
                int prior = 0;
                if (lane == 0) prior = atomicAdd(cm, 1) & 0xff;
                prior = __shfl_sync(FULL, prior, 0);
                if (prior == cur.np - 1) {
                    __threadfence_block();
                    const float4 tot = *reinterpret_cast<const float4 *>(acc);
                    *reinterpret_cast<float4 *>(p.out + row * DV + 4 * lane) =
                        make_float4(fmaf(bt[0], kq, tot.x), fmaf(bt[1], kq, tot.y),
                                    fmaf(bt[2], kq, tot.z), fmaf(bt[3], kq, tot.w));
                } else {
                    commits = false;
                }
            } else if (p.want_out) {
                *reinterpret_cast<float4 *>(p.out + row * DV + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
            }
            if (mk == MK_APPEND) {
                float *ent = ring + (size_t)c * E;
                put_seg4<LC::B16>(ent + BO, lane, bt4);
                put_seg4<LC::A16>(ent, lane, reinterpret_cast<const float4 *>(rv_k)[lane]);
                if (DECAY == DL_DECAY_DIAG)
                    *reinterpret_cast<float4 *>(ent + LO + 4 * lane) = reinterpret_cast<const float4 *>(rv_l)[lane];
                if (DECAY == DL_DECAY_SCALAR && lane == 0) ent[LO] = rv_l[0];
            } else if (mk == MK_PASS2) {
                // -- pass 2: the rows pass 1 wrote, again (from L2), plus the token term
                //    k b_t^T, row block by row block
                for (int cx = 0; cx < NCH; ++cx) {
                    if (!wait_chunk()) { abort = true; break; }
                    const float *sb = st + (size_t)(gc % NSW) * CF;
#pragma unroll
                    for (int r4 = 0; r4 < CR / 4; ++r4) {
                        const float4 k4 = reinterpret_cast<const float4 *>(rv_k + cx * CR)[r4];
                        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                        for (int y = 0; y < 4; ++y) {
                            const int rr = 4 * r4 + y;
                            float4 S = reinterpret_cast<const float4 *>(sb + rr * DV)[lane];
                            fma4(S, kv[y], bt4);
                            __stcs(reinterpret_cast<float4 *>(tile + (size_t)(cx * CR + rr) * DV) + lane, S);
                        }
                    }
                    release();
                }
                if (abort) break;
            } else if (mk == MK_ROUNDS) {
                // More entries than TMEM holds.  Pass 1 left every stage idle (no
                // look-ahead past this head).  Per round of up to MRB entries, stage 2
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
                                A[u] = seg4<LC::A16>(ent, lane);
                                B[u] = seg4<LC::B16>(ent + BO, lane);
                                if (DECAY == DL_DECAY_DIAG) {
                                    Lq[u] = ldg4(ent + LO + 4 * lane);
                                } else {
                                    const float Ls = DECAY == DL_DECAY_SCALAR ? __ldg(ent + LO) : 0.f;
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
                                const float4 l4 = reinterpret_cast<const float4 *>(rv_l)[lane];
                                const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                                const float av[4] = {A[u].x, A[u].y, A[u].z, A[u].w};
                                const float Lv[4] = {Lq[u].x, Lq[u].y, Lq[u].z, Lq[u].w};
                                float w4[4];
#pragma unroll
                                for (int x = 0; x < 4; ++x)
                                    w4[x] = DECAY == DL_DECAY_NONE ? av[x] : av[x] * expf(lv[x] - Lv[x]);
                                aw = make_float4(w4[0], w4[1], w4[2], w4[3]);
                                bw = B[u];
                            } else {
                                aw = reinterpret_cast<const float4 *>(rv_k)[lane];
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
                                const float e = rv_e[cx * CR + rr];
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
            // (a merge from an empty log leaves it empty: nothing to commit, and every
            //  unit of the slot saw the same c, so none of them counts itself in)
            if (!p.eager && commits && !(mk != MK_APPEND && c == 0)) {
                if (lane == 0) fin_old = atomicAdd(p.arrive + sl, 1);
                fin_sl = sl;
                fin_len = mk != MK_APPEND ? 0 : c + 1;
            }
        } else {
            // skipped head: nothing was streamed for it
            finish_commit();
        }

        // advance: nxt becomes cur; take the head after it and read its slot id
        if (!nxt_res) resolve_len(nxt, c_nxt);
        base += cur.n;
        cur = nxt;
        nxt.ok = 0;
        nxt.n = 0;
        it_nxt = grab(pinfo_nxt);
        s_nxt = slot_of(it_nxt, pinfo_nxt);
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
        if (use_tm) ptx::tmem_wait_st();
    }
    // tensor memory goes back once every warp is done with it
    ptx::tmem_fence_before_sync();
    __syncthreads();
    ptx::tmem_fence_after_sync();
    if (use_tm && w == 0) ptx::tmem_dealloc(*tm_slot, TM_COLS);
}

}  // namespace wh
}  // namespace dl
