// attn_kernel.cuh -- the LiteAttention step kernel for sm_100a.
//
// A FlashAttention-style forward pass over the live key/value tiles of a
// persistent skip mask, with the QK-Skip test evaluated inside the online
// softmax ("LiteAttention: Temporal Sparse Attention for Diffusion
// Transformers", Architecture Overview: QK-Skip compares a tile's max QK
// score with the cumulative max; Hardware Integration: the skip logic lives
// in the FlashAttention softmax pipeline; Persistent Propagation: decisions
// carry forward).
//
// Work item = one pair of adjacent query tiles of one (batch, head): the two
// tiles share every K/V tile load over the union of their live lists (their
// lists are near-identical under locality).  Each CTA owns 256 (Br = 128) or
// 128 (Br = 64) query rows split into "slots" of 128 rows; one tcgen05 MMA
// (M = 128) covers a slot.  With Br = 64 a slot holds both query tiles of the
// pair and rows of a tile not live for the current key tile contribute P = 0.
//
// Warp roles (128 * (1 + slots * halves) threads):
//   warp 0      TMA producer: Q of both slots once, then K_j, V_j for every
//               live entry j into a 2-stage shared-memory ring.
//   warp 1      MMA issuer (one elected lane): S_s = Q_s K_j^T into TMEM,
//               and O_s += P_s V_j with P read from TMEM (aliasing S_s).
//   warp 2      Tensor Memory allocator.
//   warps 4..   softmax.  With Bc = 128 each query row has two threads in
//               two warpgroups ("halves"), each owning 64 of the row's S
//               columns and 64 of its O columns; with Bc = 64 one warpgroup,
//               one thread per row.  Per live tile: row max (pass 1 over S),
//               QK-Skip vote (bar.red.or over the query tile's threads, which
//               also exchanges the halves' partial maxima), lazy O rescale,
//               exp2 (pass 2 over S), P -> TMEM; at the end the epilogue.
// Pipeline per entry e: PV_s(e) is issued as soon as P_s(e) is ready and is
// followed by QK_s(e+1), so each slot's softmax overlaps the other slot's
// MMAs.
//
// Every wait on an mbarrier is bounded (globaltimer); on expiry the CTA sets
// the plan's status word, stops waiting, keeps every named barrier balanced,
// drains its own copies and MMAs (bounded), frees TMEM and exits.
#pragma once

#include <cuda_bf16.h>

#include "liteattn_internal.cuh"
#include "sm100_ptx.cuh"

#ifndef LITE_HALVES
#define LITE_HALVES 2
#endif

namespace lite {

// Optional per-CTA cycle counters (compile with -DLITE_PROFILE; never in the
// product build): where each role spends its time.
#ifdef LITE_PROFILE
constexpr int kProfCtas = 65536, kProfFields = 16;
__device__ unsigned long long g_lite_prof[kProfCtas * kProfFields];
// event trace of CTA 0: [event kind][slot][entry] clock64 stamps (first kTraceEntries entries)
constexpr int kTraceEntries = 32, kTraceKinds = 8;
__device__ long long g_lite_trace[kTraceKinds * 2 * kTraceEntries];
#define LITE_PROF(x) x
#define LITE_TRACE(kind, slot, e) \
    do { if (blockIdx.x == 0 && (e) < kTraceEntries) g_lite_trace[((kind) * 2 + (slot)) * kTraceEntries + (e)] = clock64(); } while (0)
#else
#define LITE_PROF(x)
#define LITE_TRACE(kind, slot, e) do {} while (0)
#endif
// trace kinds: 0 softmax S ready, 1 vote done, 2 P stored (arrive), 3 MMA saw P, 4 MMA issued PV,
//              5 MMA issued QK(e) (slot), 6 producer issued K(e), 7 MMA saw K(e)

// Pairs of S columns (index i within a 64-column chunk) whose exponentials
// run on the FMA pipe: bit (i & 7) of this mask.  The rest use MUFU ex2.
#ifndef LITE_POLY_MASK
#define LITE_POLY_MASK 0x80u
#endif
constexpr uint32_t kPolyMask = LITE_POLY_MASK;

// Named barriers: 1..2 QK-Skip votes, 5..6 epilogue (per slot).
constexpr uint32_t kBarVote = 1, kBarEpi = 5;

struct AttnParams {
    const uint32_t *list;   // mask_in live lists [G][Tk]
    const int32_t *cnt;     // mask_in counts [G]
    const int32_t *order;   // mask_in work order [G]
    uint32_t *bits_out;     // mask_out bitmask [R][W]
    __nv_bfloat16 *o;       // [B][H][N][d]
    int32_t *status;        // plan status word
    int probe_wait;         // test of the timeout path: CTA 0's first softmax warp waits on a barrier nothing arrives on
    const int32_t *seq_len; // variable-length batches: [B] lengths (nullptr: every sequence has N tokens)
    const int64_t *seq_off; // [B] token offsets in packed [total][H][d] tensors
    int N, Tq, Tk, W, Gp;
    int H;                  // heads of the plan
    int Ht;                 // heads of the tensors (row strides; o points at the plan's first head)
    int bnhd;               // 0: q, k, v, o are [B][Ht][N][d]; 1: [B][N][Ht][d]
    int pair_stride;        // query tiles of a work item: pair_tiles(pair, Tq, pair_stride) (1 when BR = 64)
    float scale_log2;       // (1/sqrt(d)) * log2(e)
    float thr_raw;          // tau * sqrt(d): threshold on raw q.k differences (-inf = never skip)
    float recall_c;         // fixed-recall predicate: (1 - p) / p, the skipped mass a row may carry per unit kept
};

template <int D, int BR, int BC>
struct AttnCfg {
    static constexpr int NSLOT = 2 * BR / 128;   // 128-row MMA slots per CTA
    static constexpr int TPS = 128 / BR;         // query tiles per slot
    static constexpr int NST = 2;                // K/V ring stages
    static constexpr int DCH = D / 64;           // 128-byte swizzle chunks along d
    static constexpr int HALVES = (BC == 128) ? LITE_HALVES : 1;   // softmax threads per query row
    static constexpr int CPT = BC / HALVES;              // S columns per softmax thread
    static constexpr int DPT = D / HALVES;               // O columns per softmax thread
    static constexpr int NSOFT = NSLOT * HALVES;         // softmax warpgroups
    static constexpr int SLOT_THREADS = 128 * HALVES;    // softmax threads of one slot
    static constexpr int NTHREADS = 128 * (1 + NSOFT);
    static constexpr uint32_t REG_LAUNCH = (65536u / NTHREADS) & ~7u;
    static constexpr uint32_t REG_CTRL = 88;
    static constexpr uint32_t REG_SOFTMAX = ((REG_LAUNCH * NTHREADS - 128u * REG_CTRL) / (128u * NSOFT)) & ~7u;
    static constexpr bool SPLIT_REGS = NSOFT > 1;
    static_assert(!SPLIT_REGS || 128 * REG_CTRL + 128 * NSOFT * REG_SOFTMAX <= NTHREADS * REG_LAUNCH, "register split");
    static_assert(CPT % 64 == 0 || CPT == 64 || BC == 64, "columns per thread");
    static constexpr uint32_t Q_SLOT_BYTES = 128u * D * 2u;
    static constexpr uint32_t Q_CHUNK_BYTES = 128u * 128u;       // 128 rows x 128 B
    static constexpr uint32_t KV_BYTES = static_cast<uint32_t>(BC) * D * 2u;
    static constexpr uint32_t KV_CHUNK_BYTES = static_cast<uint32_t>(BC) * 128u;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + NSLOT * Q_SLOT_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NST * KV_BYTES;
    static constexpr uint32_t BM_OFF = V_OFF + NST * KV_BYTES;
    // per slot: partial row maxima [2 parities][HALVES][128], partial row sums at the end
    // [HALVES][128], partial row sums at each vote of the fixed-recall predicate [2][HALVES][128]
    static constexpr uint32_t XM_OFF = BM_OFF + 2u * kMaxWords * 4u;
    static constexpr uint32_t XM_FLOATS = 5u * HALVES * 128u;
    static constexpr uint32_t BAR_OFF = XM_OFF + NSLOT * XM_FLOATS * 4u;
    // q_full, k_full[NST], v_full[NST], k_empty[NST], v_empty[NST], s_full[NSLOT], p_full[NSLOT], o_full[NSLOT],
    // drain, never (no thread or copy ever arrives on it: the timeout-path test waits on it)
    static constexpr int NBAR = 3 + 4 * NST + 3 * NSLOT;
    static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8u;
    static constexpr uint32_t SMEM_BYTES = MISC_OFF + 64u + 1024u;  // + alignment slack
    static constexpr uint32_t S_COLS = BC;                           // fp32 S; P (bf16) aliases its first BC/2
    static constexpr uint32_t TMEM_USED = NSLOT * (BC + D);
    static constexpr uint32_t TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                          : TMEM_USED <= 256 ? 256 : 512;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(BC == 64 || BC == 128, "key tile");
    static_assert(BR == 64 || BR == 128, "query tile");
    static_assert(TMEM_USED <= 512, "tensor memory");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    __host__ __device__ static constexpr uint32_t s_col(int s) { return static_cast<uint32_t>(s) * BC; }
    __host__ __device__ static constexpr uint32_t o_col(int s) { return NSLOT * BC + static_cast<uint32_t>(s) * D; }
};

struct WaitCtx {
    volatile uint32_t *abort_flag;
    int32_t *status;
};

// Bounded mbarrier wait.  Returns false (without waiting) once the CTA has
// aborted, or after kWaitLimitNs, in which case it records the timeout.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const WaitCtx &w) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) return false;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*w.abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                *w.abort_flag = 1u;
                atomicExch(w.status, kStatusTimeout);
                return false;
            }
        }
    }
}
// Bounded wait used only while draining at exit (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 63u && ptx::globaltimer_ns() - t0 > kWaitLimitNs) return;
    }
}

template <int TPS>
__device__ __forceinline__ bool slot_live(uint32_t flags, int s) {
    return TPS == 1 ? ((flags >> s) & 1u) != 0u : flags != 0u;
}

// RECALL selects the skip predicate: false = the QK-Skip threshold test, true =
// the fixed-recall test ("Training-free sparse attention based on cumulative
// energy filtering", abstract: a fixed recall rate held by a dynamic threshold
// inside the FlashAttention pass).  Under the latter each row carries z, an
// upper bound on the softmax mass of the key tiles it skipped (in the frame of
// its running sum l); a live-in tile of w valid keys is skipped for the query
// tile when every valid row has z + w * e^(m_loc - m) <= c * l, c = (1 - p) / p,
// so every row keeps recall >= p.
template <int D, int BR, int BC, bool RECALL>
__global__ void __launch_bounds__(AttnCfg<D, BR, BC>::NTHREADS, 1)
lite_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = AttnCfg<D, BR, BC>;
    constexpr int NSLOT = C::NSLOT, TPS = C::TPS, NST = C::NST;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = ptx::smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);

    const uint32_t bar0 = base_s + C::BAR_OFF;
    auto q_full = [&]() { return bar0; };
    auto k_full = [&](int st) { return bar0 + 8u * (1 + st); };
    auto v_full = [&](int st) { return bar0 + 8u * (1 + NST + st); };
    auto k_empty = [&](int st) { return bar0 + 8u * (1 + 2 * NST + st); };
    auto v_empty = [&](int st) { return bar0 + 8u * (1 + 3 * NST + st); };
    auto s_full = [&](int s) { return bar0 + 8u * (1 + 4 * NST + s); };
    auto p_full = [&](int s) { return bar0 + 8u * (1 + 4 * NST + NSLOT + s); };
    auto o_full = [&](int s) { return bar0 + 8u * (1 + 4 * NST + 2 * NSLOT + s); };
    const uint32_t drain = o_full(0) + 8u * NSLOT;
    const uint32_t never = drain + 8u;

    uint32_t *misc = reinterpret_cast<uint32_t *>(base + C::MISC_OFF);
    volatile uint32_t *tmem_slot = misc + 0;
    volatile uint32_t *abort_flag = misc + 1;
    volatile uint32_t *pvf = misc + 2;  // [2] live-now flag per query tile of the pair
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(base + C::BM_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#ifdef LITE_DEBUG_CHECKS
    // Debug builds: check this CTA's work item before using it.  A bad one is
    // recorded in the status word and processed as an empty item (nothing is read
    // through it), so a corrupt order, count or list never sends an access out of
    // bounds.
    int grp = p.order[blockIdx.x];
    const bool grp_ok = grp >= 0 && grp < static_cast<int>(gridDim.x);
    if (!grp_ok) grp = 0;
    int n_e = p.cnt[grp];
    {
        bool bad = !grp_ok || n_e < 0 || n_e > p.Tk;
        if (bad) n_e = 0;
        int qa_chk, qb_chk;
        pair_tiles(grp % p.Gp, p.Tq, p.pair_stride, qa_chk, qb_chk);
        const uint32_t *el = p.list + static_cast<int64_t>(grp) * p.Tk;
        for (int e = threadIdx.x; !bad && e < n_e; e += C::NTHREADS) {
            const uint32_t x = __ldg(el + e);
            const int j = static_cast<int>(x & kEntryMask);
            const uint32_t f = x >> kFlagShift;
            const bool prev_ok = e == 0 || static_cast<int>(__ldg(el + e - 1) & kEntryMask) < j;
            const bool flags_ok = f != 0u && ((f & 2u) == 0u || qb_chk >= 0);
            if (j >= p.Tk || !prev_ok || !flags_ok) bad = true;
        }
        if (__syncthreads_or(bad ? 1 : 0)) {
            if (threadIdx.x == 0) atomicExch(p.status, kStatusCheck);
            n_e = 0;
        }
    }
#else
    const int grp = p.order[blockIdx.x];
    const int n_e = p.cnt[grp];
#endif
    const int bh = grp / p.Gp, pr = grp % p.Gp;
    int qt0, qt1;   // the pair's query tiles (qt1 = -1: none)
    pair_tiles(pr, p.Tq, p.pair_stride, qt0, qt1);
    // this work item's sequence: its length, query and key tile counts, and where its
    // tokens start (variable-length batches are packed token-major, [total][H][d])
    const int b_seq = bh / p.H;
    const int Nb = p.seq_len ? p.seq_len[b_seq] : p.N;
    const int Tqb = (Nb + BR - 1) / BR, Tkb = (Nb + BC - 1) / BC;
    const int64_t tok0 = p.seq_len ? p.seq_off[b_seq] : static_cast<int64_t>(b_seq) * p.N;
    const uint32_t *elist = p.list + static_cast<int64_t>(grp) * p.Tk;
    const WaitCtx wctx{abort_flag, p.status};
    LITE_PROF(const long long prof_t_start = clock64(); unsigned long long prof[kProfFields] = {};)

    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full(), 1);
        for (int st = 0; st < NST; ++st) {
            ptx::mbar_init(k_full(st), 1);
            ptx::mbar_init(v_full(st), 1);
            ptx::mbar_init(k_empty(st), 1);
            ptx::mbar_init(v_empty(st), 1);
        }
        for (int s = 0; s < NSLOT; ++s) {
            ptx::mbar_init(s_full(s), 1);
            ptx::mbar_init(p_full(s), C::SLOT_THREADS);
        }
        for (int s = 0; s < NSLOT; ++s) ptx::mbar_init(o_full(s), 1);
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(never, 1);
        *abort_flag = 0u;
        pvf[0] = 0u;
        pvf[1] = 0u;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_u32(misc), C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp >= 4) {  // softmax warpgroups clear the bitmap rows of their query tiles
        const int g = warp / 4 - 1, wg = g / C::HALVES;
        const int idx = (g % C::HALVES) * 128 + (threadIdx.x & 127);
        const int t_lo = (TPS == 1) ? wg : 0, t_hi = (TPS == 1) ? wg : 1;
        for (int t = t_lo; t <= t_hi; ++t)
            for (int w = idx; w < p.W; w += C::SLOT_THREADS) bitmap[t * kMaxWords + w] = 0u;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Register split: the launch gives NTHREADS x 168 registers; the control
    // warpgroup drops to REG_CTRL and the softmax warpgroups rise to
    // REG_SOFTMAX (128*REG_CTRL + 256*REG_SOFTMAX <= 384*168, checked above).
    if (warp < 4) {
      if constexpr (C::SPLIT_REGS) ptx::regs_dec<C::REG_CTRL>();
      if (warp == 0) {
        // ============================================================ TMA producer
        // The whole warp runs the loop (uniform operands); one elected lane issues.
        // The tensor maps are 4-D: (d, N, H, B) for [B][H][N][d] tensors and
        // (d, H, N, B) for [B][N][H][d]; a box is 64 elements of d by `rows` tokens
        // of one (batch, head), so shared memory sees the same tile either way.
        // Variable-length batches use (d, H, total tokens, 1) maps: token tok0 + row.
        const int b_idx = bh / p.H, h_idx = bh % p.H;
        auto load_rows = [&](uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int row) {
            if (p.seq_len) ptx::tma_load_4d_elect(dst, m, bar, x, h_idx, static_cast<int>(tok0) + row, 0);
            else if (p.bnhd) ptx::tma_load_4d_elect(dst, m, bar, x, h_idx, row, b_idx);
            else ptx::tma_load_4d_elect(dst, m, bar, x, row, h_idx, b_idx);
        };
        // slot s holds query tile qt_s (BR = 128), or both tiles of the pair, which are
        // adjacent then, from qt0 on (BR = 64)
        auto slot_tile = [&](int s) { return s == 0 ? qt0 : qt1; };
        auto slot_loaded = [&](int s) { return (TPS == 2) || (slot_tile(s) >= 0 && slot_tile(s) < Tqb); };
        uint32_t qbytes = 0;
        for (int s = 0; s < NSLOT; ++s)
            if (slot_loaded(s)) qbytes += C::Q_SLOT_BYTES;
        ptx::mbar_arrive_expect_tx_elect(q_full(), qbytes);
        for (int s = 0; s < NSLOT; ++s) {
            if (!slot_loaded(s)) continue;
            const int row0 = slot_tile(s) * BR;
            for (int c = 0; c < C::DCH; ++c)
                load_rows(base_s + C::Q_OFF + s * C::Q_SLOT_BYTES + c * C::Q_CHUNK_BYTES, &tm_q, q_full(), c * 64, row0);
        }
        int issued = 0;
        for (int e = 0; e < n_e; ++e) {
            const int st = e % NST;
            const uint32_t ph = (e / NST) & 1;
            const int j = static_cast<int>(__ldg(elist + e) & kEntryMask);
            // K(e) may enter its stage once QK of entry e-NST completed, V(e) once PV of e-NST did
            LITE_PROF(long long tk = clock64();)
            if (!__all_sync(0xFFFFFFFFu, wait_bar(k_empty(st), ph ^ 1u, wctx))) break;
            LITE_PROF(prof[13] += clock64() - tk;)
            if (lane == 0) LITE_TRACE(6, 0, e);
            ptx::mbar_arrive_expect_tx_elect(k_full(st), C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
                load_rows(base_s + C::K_OFF + st * C::KV_BYTES + c * C::KV_CHUNK_BYTES, &tm_k, k_full(st), c * 64, j * BC);
            LITE_PROF(long long tv = clock64();)
            const bool v_ok = __all_sync(0xFFFFFFFFu, wait_bar(v_empty(st), ph ^ 1u, wctx));
            LITE_PROF(prof[14] += clock64() - tv;)
            if (!v_ok) {
                issued = e;   // K(e) is in flight: drain it below
                drain_wait(k_full(st), ph);
                break;
            }
            ptx::mbar_arrive_expect_tx_elect(v_full(st), C::KV_BYTES);
            for (int c = 0; c < C::DCH; ++c)
                load_rows(base_s + C::V_OFF + st * C::KV_BYTES + c * C::KV_CHUNK_BYTES, &tm_v, v_full(st), c * 64, j * BC);
            issued = e + 1;
        }
        // drain: every copy this CTA started must land before it exits
        drain_wait(q_full(), 0);
        for (int e = (issued > NST ? issued - NST : 0); e < issued; ++e) {
            drain_wait(k_full(e % NST), (e / NST) & 1);
            drain_wait(v_full(e % NST), (e / NST) & 1);
        }
        __syncwarp();
      } else if (warp == 1) {
        // ============================================================ MMA issuer
        // The whole warp runs the loop so that descriptors and TMEM addresses
        // stay warp-uniform; one elected lane issues each block of tcgen05 MMAs
        // and each commit.
        constexpr uint32_t IDESC_QK = ptx::idesc_bf16_f32(128, BC, false);
        constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, D, true);
        // Shared-memory descriptors are built once; each MMA adds a compile-time
        // offset (16-byte units) to the start-address field, which cannot carry
        // out of its 14 bits (shared addresses < 256 KB).
        const uint64_t dq0 = ptx::sdesc_sw128(base_s + C::Q_OFF, 16, 1024);
        const uint64_t dk0 = ptx::sdesc_sw128(base_s + C::K_OFF, 16, 1024);
        const uint64_t dv0 = ptx::sdesc_sw128(base_s + C::V_OFF, C::KV_CHUNK_BYTES, 1024);
        auto issue_qk = [&](int s, int st) {
            const uint64_t qa = dq0 + ((s * C::Q_SLOT_BYTES) >> 4);
            const uint64_t ka = dk0 + ((st * C::KV_BYTES) >> 4);
            const uint32_t d = tmem + C::s_col(s);
            if (ptx::elect_one()) {   // one lane issues the whole block of MMAs
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off_q = ((kk >> 2) * C::Q_CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t off_k = ((kk >> 2) * C::KV_CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    ptx::mma_ss(d, qa + off_q, ka + off_k, IDESC_QK, kk > 0 ? 1u : 0u);
                }
            }
            __syncwarp();
        };
        auto issue_pv = [&](int s, int st, bool first) {
            const uint64_t va = dv0 + ((st * C::KV_BYTES) >> 4);
            const uint32_t d = tmem + C::o_col(s), a = tmem + C::s_col(s);
            // P of keys [h*CPT, (h+1)*CPT) sits in TMEM columns [h*CPT, h*CPT + CPT/2) of the slot's S
            // region (written by the softmax thread that owns those columns); 16 keys per MMA = 8 columns
            if (ptx::elect_one()) {
#pragma unroll
                for (int kk = 0; kk < BC / 16; ++kk) {
                    const uint32_t pc = (kk / (C::CPT / 16)) * C::CPT + (kk % (C::CPT / 16)) * 8;
                    ptx::mma_ts(d, a + pc, va + ((kk * 16 * 128) >> 4), IDESC_PV, (first && kk == 0) ? 0u : 1u);
                }
            }
            __syncwarp();
        };
        auto wait_all = [&](uint32_t bar, uint32_t par) { return __all_sync(0xFFFFFFFFu, wait_bar(bar, par, wctx)); };
        bool ok = wait_all(q_full(), 0);
        LITE_PROF(const long long tm0 = clock64(); prof[15] = tm0 - prof_t_start;)
        uint32_t pph[NSLOT];
        bool first[NSLOT];
        for (int s = 0; s < NSLOT; ++s) {
            pph[s] = 0;
            first[s] = true;
        }
        if (n_e > 0) {
            const uint32_t f0 = __ldg(elist) >> kFlagShift;
            ok = wait_all(k_full(0), 0) && ok;
            ptx::tc_fence_after();
            for (int s = 0; s < NSLOT; ++s)
                if (slot_live<TPS>(f0, s)) {
                    if (ok) issue_qk(s, 0);
                    ptx::mma_commit_elect(s_full(s));
                    if (lane == 0) LITE_TRACE(5, s, 0);
                }
            ptx::mma_commit_elect(k_empty(0));
        }
        for (int e = 0; e < n_e; ++e) {
            const int st = e % NST;
            const uint32_t ph = (e / NST) & 1;
            const uint32_t f = __ldg(elist + e) >> kFlagShift;
            const bool has_next = (e + 1) < n_e;
            const uint32_t f1 = has_next ? (__ldg(elist + e + 1) >> kFlagShift) : 0u;
            const int st1 = (e + 1) % NST;
            const uint32_t ph1 = ((e + 1) / NST) & 1;
            bool v_ready = false, k1_ready = false;
            for (int s = 0; s < NSLOT; ++s) {
                if (slot_live<TPS>(f, s)) {
                    LITE_PROF(long long t0 = clock64();)
                    ok = wait_all(p_full(s), pph[s]) && ok;
                    LITE_PROF(prof[1] += clock64() - t0;)
                    if (lane == 0) LITE_TRACE(3, s, e);
                    pph[s] ^= 1u;
                    ptx::tc_fence_after();
                    const bool pv = (TPS == 1) ? (pvf[s] != 0u) : ((pvf[0] | pvf[1]) != 0u);
                    if (pv) {
                        if (!v_ready) {
                            LITE_PROF(long long t1 = clock64();)
                            ok = wait_all(v_full(st), ph) && ok;
                            LITE_PROF(prof[3] += clock64() - t1;)
                            v_ready = true;
                        }
                        if (ok) issue_pv(s, st, first[s]);
                        if (lane == 0) LITE_TRACE(4, s, e);
                        first[s] = false;
                    }
                }
                if (has_next && slot_live<TPS>(f1, s)) {
                    if (!k1_ready) {
                        LITE_PROF(long long t2 = clock64();)
                        ok = wait_all(k_full(st1), ph1) && ok;
                        LITE_PROF(prof[2] += clock64() - t2;)
                        if (lane == 0) LITE_TRACE(7, 0, e + 1);
                        k1_ready = true;
                        ptx::tc_fence_after();
                    }
                    if (ok) issue_qk(s, st1);
                    ptx::mma_commit_elect(s_full(s));
                    if (lane == 0) LITE_TRACE(5, s, e + 1);
                }
                // after the slot's part of the last entry its O is final: its epilogue
                // may start while the other slot finishes
                if (!has_next) ptx::mma_commit_elect(o_full(s));
            }
            if (has_next) ptx::mma_commit_elect(k_empty(st1));
            if (!v_ready) ok = wait_all(v_full(st), ph) && ok;
            ptx::mma_commit_elect(v_empty(st));
        }
        if (n_e == 0)
            for (int s = 0; s < NSLOT; ++s) ptx::mma_commit_elect(o_full(s));
        LITE_PROF(prof[4] = clock64() - tm0;)
        ptx::mma_commit_elect(drain);
        drain_wait(drain, 0);
        __syncwarp();
      }
    } else {
        // ============================================================ softmax warpgroups
        if constexpr (C::SPLIT_REGS) ptx::regs_inc<C::REG_SOFTMAX>();
        // Test of the timeout path only: a wait that runs out after kWaitLimitNs, sets
        // the status word and sends the whole CTA down its abort path.
        if (p.probe_wait && blockIdx.x == 0 && warp == 4) (void)wait_bar(never, 0, wctx);
        constexpr int HALVES = C::HALVES, CPT = C::CPT, DPT = C::DPT;
        const int g = warp / 4 - 1;         // softmax warpgroup
        const int wg = g / HALVES;          // slot
        const int half = g % HALVES;        // which columns of the row this thread owns
        const int wq = warp & 3;            // TMEM lane quarter
        const int r = wq * 32 + lane;       // row within the slot (TMEM lane)
        const int rig = wg * 128 + r;       // row within the pair
        const int t = rig / BR;             // query tile of the pair (0/1)
        const int qt = t ? qt1 : qt0;
        const int n = qt >= 0 ? qt * BR + rig % BR : 0;   // token index
        const bool row_valid = (qt >= 0) && (qt < Tqb) && (n < Nb);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t scol = C::s_col(wg) + half * CPT;        // this thread's S columns (fp32)
        const uint32_t pcol = C::s_col(wg) + half * CPT;        // its P columns: bf16 pairs over its own S
        const uint32_t ocol = C::o_col(wg) + half * DPT;        // its O columns
        const uint32_t vote_bar = (TPS == 1) ? kBarVote + wg : kBarVote + t;
        const uint32_t vote_n = (TPS == 1) ? C::SLOT_THREADS : 64u;
        const bool leader = half == 0 && (rig % BR) == 0;
        uint32_t *bm = bitmap + t * kMaxWords;
        // partial row maxima (and, at the end, row sums) exchanged between the two halves of a row
        float *xm = reinterpret_cast<float *>(base + C::XM_OFF) + wg * C::XM_FLOATS;
        float *xl = xm + 2 * HALVES * 128;
        float *xlv = xm + 3 * HALVES * 128;   // fixed-recall votes: partial row sums [2 parities][HALVES][128]
        const float cl2 = p.scale_log2;
        const float thr = p.thr_raw;
        const float resc_thr = 8.0f / cl2;  // lazy-rescale trigger: running max grew by > 2^8 in weight
        float m_run = -INFINITY, m_ref = -INFINITY, l = 0.0f;
        float z = 0.0f;   // fixed-recall predicate: skipped-mass bound of the row, frame of l (both halves alike)
        float lx = 0.0f;  // fixed-recall predicate: this half's kept mass from the unrounded weights (frame of l)
        uint32_t sph = 0;
        const int tail = Nb - (Tkb - 1) * BC;  // valid columns of the sequence's last key tile

        uint32_t ent_next = (n_e > 0) ? __ldg(elist) : 0u;  // list entries are read one ahead
        for (int e = 0; e < n_e; ++e) {
            const uint32_t ent = ent_next;
            if (e + 1 < n_e) ent_next = __ldg(elist + e + 1);
            const uint32_t f = ent >> kFlagShift;
            if (!slot_live<TPS>(f, wg)) continue;
            const int j = static_cast<int>(ent & kEntryMask);
            const bool tile_in = (TPS == 1) ? true : (((f >> t) & 1u) != 0u);
            LITE_PROF(long long ts0 = clock64();)
            bool ok = wait_bar(s_full(wg), sph, wctx);
            LITE_PROF(long long ts1 = clock64(); if (g == 0) { prof[5] += ts1 - ts0; prof[8] += 1; })
            if ((threadIdx.x & 127) == 0 && half == 0) LITE_TRACE(0, wg, e);
            const uint32_t par = sph;
            sph ^= 1u;
            ok = __all_sync(0xFFFFFFFFu, ok);
            ptx::tc_fence_after();

            // Pass 1 over this thread's S columns: the row maximum.  The values die
            // here; pass 2 reads them from TMEM again, 32 columns at a time, which
            // keeps the register footprint small enough for two threads per row.
            const bool tail_tile = (j == Tkb - 1) && (tail < BC);
            float m_part;
            {
                // 8 independent 3-input max chains, fed 32 columns at a time
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
                for (int ch = 0; ch < CPT / 32; ++ch) {
                    uint32_t sr[32];
                    if (ok) {
                        ptx::tmem_ld32(lane_base + scol + ch * 32, sr);
                        ptx::tmem_ld_wait(sr);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) sr[i] = 0u;
                    }
                    if (tail_tile) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (half * CPT + ch * 32 + i >= tail) sr[i] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int c = 0; c < 32; c += 16)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mx[k] = ptx::max3(mx[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
                }
                LITE_PROF(if (g == 0) prof[9] += clock64() - ts1;)
                m_part = ptx::max3(ptx::max3(mx[0], mx[1], mx[2]), ptx::max3(mx[3], mx[4], mx[5]),
                                   fmaxf(mx[6], mx[7]));
            }
            if (HALVES == 2) xm[(par * HALVES + half) * 128 + r] = m_part;
            LITE_PROF(long long tmx = clock64();)

            const bool active = row_valid && tile_in;
            bool live;
            float m_loc, ub = 0.0f;
            if constexpr (!RECALL) {
                // QK-Skip: the tile stays live for this query tile if any valid row rose
                // by at least tau over its running max.  max(a, b) - m >= tau iff either
                // half does, so one barrier reduction over both halves decides, and it
                // also publishes the partial maxima.
                const bool want = active && (m_part - m_run >= thr);
                live = ptx::bar_red_or(vote_bar, vote_n, want);
                m_loc = (HALVES == 2) ? fmaxf(m_part, xm[(par * HALVES + (half ^ 1)) * 128 + r]) : m_part;
            } else {
                // Fixed recall: the row's test needs its whole max and whole kept mass, so
                // the halves first exchange both (one barrier), then vote (a second).
                // the budget uses the kept mass summed from the unrounded weights, as the
                // predicate defines it (l itself adds the bf16 weights that P.V consumes)
                float l_row = lx;
                if (HALVES == 2) {
                    xlv[(par * HALVES + half) * 128 + r] = lx;
                    ptx::bar_sync(vote_bar, vote_n);
                    m_loc = fmaxf(m_part, xm[(par * HALVES + (half ^ 1)) * 128 + r]);
                    l_row += xlv[(par * HALVES + (half ^ 1)) * 128 + r];
                } else {
                    m_loc = m_part;
                }
                // the tile's mass bound for this row: valid keys x peak weight, frame of l
                // (+inf before the row's first kept tile, when m_ref = -inf)
                const float w = tail_tile ? static_cast<float>(tail) : static_cast<float>(BC);
                ub = w * ptx::ex2((m_loc - m_ref) * cl2);
                const bool afford = z + ub <= p.recall_c * l_row;
                live = ptx::bar_red_or(vote_bar, vote_n, active && !afford);
                if (active && !live && m_ref > -INFINITY) z += ub;   // skipped: its bound joins z
            }
            LITE_PROF(long long ts2 = clock64(); if (g == 0) { prof[6] += ts2 - ts1; prof[10] += ts2 - tmx; })
            if ((threadIdx.x & 127) == 0 && half == 0) LITE_TRACE(1, wg, e);
            if (leader) {
                const bool lv = tile_in && live;
                pvf[t] = lv ? 1u : 0u;
                if (lv) bm[j >> 5] |= (1u << (j & 31));
            }
            __syncwarp();
            if (TPS == 1 && !live) {  // dead for this query tile: no softmax, no PV
                ptx::tc_fence_before();
                ptx::mbar_arrive(p_full(wg));
                continue;
            }
            const bool do_p = active && live;
            bool need_rescale = false;
            float alpha = 1.0f;
            if (do_p) {
                const float m_new = fmaxf(m_run, m_loc);
                m_run = m_new;
                if (m_new - m_ref > resc_thr) {
                    if (l > 0.0f) {
                        alpha = ptx::ex2((m_ref - m_new) * cl2);
                        need_rescale = true;
                        l *= alpha;
                    }
                    // z and lx move to the new frame with l (both are 0 while m_ref = -inf)
                    if constexpr (RECALL) {
                        const float a = ptx::ex2((m_ref - m_new) * cl2);
                        z *= a;
                        lx *= a;
                    }
                    m_ref = m_new;
                }
            }
            if (__any_sync(0xFFFFFFFFu, need_rescale) && ok) {
                const uint64_t a2 = ptx::f2(alpha, alpha);
#pragma unroll 1
                for (int ch = 0; ch < DPT / 16; ++ch) {
                    uint32_t orow[16];
                    ptx::tmem_ld16(lane_base + ocol + ch * 16, orow);
                    ptx::tmem_ld_wait16(orow);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float a, b;
                        ptx::f2_split(ptx::mul2(ptx::f2(__uint_as_float(orow[2 * i]), __uint_as_float(orow[2 * i + 1])),
                                                a2), a, b);
                        orow[2 * i] = __float_as_uint(a);
                        orow[2 * i + 1] = __float_as_uint(b);
                    }
                    ptx::tmem_st16(lane_base + ocol + ch * 16, orow);
                }
            }
            // P = 2^(s*scale*log2e - m_ref*scale*log2e); rows not taking part get -inf -> 0.
            const float neg = do_p ? -m_ref * cl2 : -INFINITY;
            const uint64_t c2 = ptx::f2(cl2, cl2), n2 = ptx::f2(neg, neg);
            // The row sum adds the bf16-rounded weights that the P.V MMA consumes, so
            // the output is a weighted mean whose numerator and denominator use the
            // same weights (a weight's rounding scales both).  Mixed-precision
            // f32 += bf16 adds, 8 independent partial sums.
            float accs[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) accs[k] = 0.0f;
            uint64_t accx[2] = {ptx::f2(0.0f, 0.0f), ptx::f2(0.0f, 0.0f)};   // fixed-recall plans: unrounded weights
            // Pass 2, 32 columns at a time: 16 packed bf16 pairs per TMEM store.
#pragma unroll
            for (int ch = 0; ch < CPT / 32; ++ch) {
                uint32_t sc[32];
                if (ok) {
                    ptx::tmem_ld32(lane_base + scol + ch * 32, sc);
                    ptx::tmem_ld_wait(sc);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) sc[i] = 0u;
                }
                if (tail_tile) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (half * CPT + ch * 32 + i >= tail) sc[i] = __float_as_uint(-INFINITY);
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float x0, x1, p0, p1;
                    ptx::f2_split(ptx::fma2(ptx::f2(__uint_as_float(sc[2 * i]), __uint_as_float(sc[2 * i + 1])), c2, n2),
                                  x0, x1);
                    if ((kPolyMask >> (i & 7)) & 1u) {
                        ptx::exp2_poly2(x0, x1, p0, p1);
                    } else {
                        p0 = ptx::ex2(x0);
                        p1 = ptx::ex2(x1);
                    }
                    pk[i] = ptx::pack_bf16x2(p0, p1);
                    ptx::add_bf16x2(accs[2 * (i & 3)], accs[2 * (i & 3) + 1], pk[i]);
                    if constexpr (RECALL) accx[i & 1] = ptx::add2(accx[i & 1], ptx::f2(p0, p1));
                }
                if (ok) ptx::tmem_st16(lane_base + pcol + ch * 16, pk);
            }
            if (do_p) l += ((accs[0] + accs[1]) + (accs[2] + accs[3])) + ((accs[4] + accs[5]) + (accs[6] + accs[7]));
            if constexpr (RECALL) {
                float x0, x1;
                ptx::f2_split(ptx::add2(accx[0], accx[1]), x0, x1);
                if (do_p) lx += x0 + x1;
            }
            LITE_PROF(long long tst = clock64();)
            ptx::tmem_st_wait();
            LITE_PROF(if (g == 0) prof[11] += clock64() - tst;)
            ptx::tc_fence_before();
            ptx::mbar_arrive(p_full(wg));
            if ((threadIdx.x & 127) == 0 && half == 0) LITE_TRACE(2, wg, e);
            LITE_PROF(if (g == 0) prof[7] += clock64() - ts2;)
        }

        // ---------------------------------------------------------------- epilogue
        LITE_PROF(const long long te0 = clock64();)
        // row sums of the two halves
        if (HALVES == 2) xl[half * 128 + r] = l;
        ptx::bar_sync(kBarEpi + wg, C::SLOT_THREADS);
        if (HALVES == 2) l += xl[(half ^ 1) * 128 + r];
        bool ok = wait_bar(o_full(wg), 0, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        ptx::tc_fence_after();
        const bool has_l = l > 0.0f;
        const float inv_l = has_l ? 1.0f / l : 0.0f;
        const int64_t orow_idx = p.bnhd ? (tok0 + n) * p.Ht + bh % p.H
                                        : (static_cast<int64_t>(bh / p.H) * p.Ht + bh % p.H) * p.N + n;
        __nv_bfloat16 *orow_g = p.o + orow_idx * D + half * DPT;
#pragma unroll 1
        for (int ch = 0; ch < DPT / 16; ++ch) {
            uint32_t ov[16];
            if (ok) {
                ptx::tmem_ld16(lane_base + ocol + ch * 16, ov);
                ptx::tmem_ld_wait16(ov);
            }
            if (row_valid) {
                uint32_t pk[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float a = 0.0f, b = 0.0f;
                    if (has_l && ok)
                        ptx::f2_split(ptx::mul2(ptx::f2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1])),
                                                ptx::f2(inv_l, inv_l)), a, b);
                    pk[i] = ptx::pack_bf16x2(a, b);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(orow_g + ch * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        LITE_PROF(prof[12] = clock64() - te0;)
        // mask_out rows of this slot's query tiles (the bitmap is complete: every
        // decision was recorded before the slot's last barrier above)
        const int t_lo = (TPS == 1) ? wg : 0, t_hi = (TPS == 1) ? wg : 1;
        for (int tt = t_lo; tt <= t_hi; ++tt) {
            const int q2 = tt ? qt1 : qt0;
            if (q2 < 0 || q2 >= p.Tq) continue;
            uint32_t *dst = p.bits_out + (static_cast<int64_t>(bh) * p.Tq + q2) * p.W;
            for (int w = half * 128 + r; w < p.W; w += C::SLOT_THREADS) dst[w] = bitmap[tt * kMaxWords + w];
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 2) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
#ifdef LITE_PROFILE
    if (blockIdx.x < kProfCtas) {
        unsigned long long *dst = g_lite_prof + static_cast<size_t>(blockIdx.x) * kProfFields;
        if (threadIdx.x == 32) for (int i = 1; i <= 4; ++i) dst[i] = prof[i];
        if (threadIdx.x == 32) dst[15] = prof[15];
        if (threadIdx.x == 0) { dst[13] = prof[13]; dst[14] = prof[14]; }
        if (threadIdx.x == 128) { for (int i = 5; i <= 8; ++i) dst[i] = prof[i]; dst[12] = prof[12];
                                  dst[0] = clock64() - prof_t_start; }
        if (threadIdx.x == 128) for (int i = 9; i <= 11; ++i) dst[i] = prof[i];
    }
#endif
}

}  // namespace lite
