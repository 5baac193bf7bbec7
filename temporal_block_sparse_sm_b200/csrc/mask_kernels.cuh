// mask_kernels.cuh -- skip-mask store kernels: reset to all-live, and
// compaction of the bitmask into per-query-tile-pair live lists.
//
// The mask holds the pages' two forms of the Skip-Mask ("LiteAttention:
// Temporal Sparse Attention for Diffusion Transformers", Architecture
// Overview: a bitmask, or a skip-list for high sparsity).  The attention
// kernel writes the bitmask; this compaction turns it into the list form the
// next step's attention kernel walks, so dead tiles are never touched.
//
// Both kernels are memory-bound: the compaction reads R*W words and writes
// one 4-byte entry per live (pair, key tile) plus 8 bytes per pair.
#pragma once

#include "liteattn_internal.cuh"

namespace lite {

// Every valid tile live: bits, lists (0..Tk-1 with both pair flags where the
// second query tile exists; pairs as pair_tiles), counts = Tk, identity order, stats.  In a
// variable-length batch, "valid" is per sequence: query tiles [0, Tq_b) and key
// tiles [0, Tk_b) of sequence b; its other rows and bits are dead.
__global__ void mask_reset_kernel(MaskDev m, Geometry g) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t nbits = g.R * g.W;
    for (int64_t idx = tid; idx < nbits; idx += nthr) {
        const int w = static_cast<int>(idx % g.W);
        const int64_t row = idx / g.W;
        const int i = static_cast<int>(row % g.Tq);
        const int Nb = seq_length(g, static_cast<int>(row / g.Tq) / g.H);
        const int Tqb = (Nb + g.Br - 1) / g.Br, Tkb = (Nb + g.Bc - 1) / g.Bc;
        const int lo = w * 32, nvalid = Tkb - lo;    // key tiles of this word that exist
        uint32_t word = 0u;
        if (i < Tqb && nvalid > 0) word = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
        m.bits[idx] = word;
    }
    const int64_t nlist = static_cast<int64_t>(g.G) * g.Tk;
    for (int64_t idx = tid; idx < nlist; idx += nthr) {
        const int grp = static_cast<int>(idx / g.Tk);
        const int e = static_cast<int>(idx % g.Tk);
        const int pr = grp % g.Gp;
        const int Nb = seq_length(g, (grp / g.Gp) / g.H);
        const int Tqb = (Nb + g.Br - 1) / g.Br;
        int qa, qb;
        pair_tiles(pr, g.Tq, g.pair_stride, qa, qb);
        const uint32_t second = (qb >= 0 && qb < Tqb) ? 2u : 0u;
        m.list[idx] = static_cast<uint32_t>(e) | ((1u | second) << kFlagShift);
    }
    for (int64_t idx = tid; idx < g.G; idx += nthr) {
        const int pr = static_cast<int>(idx % g.Gp);
        const int Nb = seq_length(g, static_cast<int>(idx / g.Gp) / g.H);
        const int Tqb = (Nb + g.Br - 1) / g.Br, Tkb = (Nb + g.Bc - 1) / g.Bc;
        int qa, qb;
        pair_tiles(pr, g.Tq, g.pair_stride, qa, qb);
        m.cnt[idx] = (qa < Tqb) ? Tkb : 0;
        m.order[idx] = static_cast<int32_t>(idx);
    }
    if (tid == 0) {
        m.stats->live = g.tiles_total;
        m.stats->live_in = 0;
        m.stats->newly_dead = 0;
        m.stats->last_step = -1;
        *m.done = 0u;
    }
}

constexpr int kCompactWarps = 8;               // warps per compaction block, one pair per warp
constexpr int kCompactThreads = 32 * kCompactWarps;
constexpr int kOrderBuckets = 1024;               // multiple of kCompactThreads

// Bitmask -> live lists.  One warp per query-tile pair (tiles as pair_tiles); lane w handles word
// w (+32k) of both rows; a warp-wide exclusive scan of the per-word counts
// gives each lane its output offset, so entries come out in ascending j.
// The last block to finish (threadfence + counter, no spinning) totals the
// live count, writes the stats, and builds the longest-first work order with
// a counting sort over (coarsened) counts (or the head-by-head index order,
// for plans whose per-head K and V do not fit a quarter of L2).
//   step_mode: 1 = called after a step (live_in_src = incoming mask's live
//   count, read before it may be overwritten), 0 = after an import.
__global__ void __launch_bounds__(kCompactThreads)
mask_compact_kernel(MaskDev m, Geometry g, int step_mode, const MaskStats *live_in_src, int step,
                    PlanDev *plan) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = blockIdx.x * kCompactWarps + warp;
    long long live = 0;
    if (grp < g.G) {
        const int bh = grp / g.Gp, pr = grp % g.Gp;
        int qa, qb;
        pair_tiles(pr, g.Tq, g.pair_stride, qa, qb);
        const bool has1 = qb >= 0;
        const uint32_t *b0 = m.bits + (static_cast<int64_t>(bh) * g.Tq + qa) * g.W;
        const uint32_t *b1 = m.bits + (static_cast<int64_t>(bh) * g.Tq + (has1 ? qb : qa)) * g.W;
        uint32_t *out = m.list + static_cast<int64_t>(grp) * g.Tk;
        // bits >= Tk are ignored even if a caller's bitmask sets them, so a list never
        // holds more than Tk entries
        const uint32_t last_keep = (g.Tk & 31) ? ((1u << (g.Tk & 31)) - 1u) : 0xFFFFFFFFu;
        int base = 0;
        for (int w0 = 0; w0 < g.W; w0 += 32) {
            const int w = w0 + lane;
            const uint32_t keep = (w == g.W - 1) ? last_keep : 0xFFFFFFFFu;
            const uint32_t a = (w < g.W) ? (b0[w] & keep) : 0u;
            const uint32_t b = (w < g.W && has1) ? (b1[w] & keep) : 0u;
            uint32_t u = a | b;
            const int c = __popc(u);
            live += __popc(a) + __popc(b);
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += y;
            }
            int pos = base + incl - c;
            while (u) {
                const int bit = __ffs(u) - 1;
                u &= u - 1u;
                const uint32_t flags = ((a >> bit) & 1u) | (((b >> bit) & 1u) << 1);
                out[pos++] = static_cast<uint32_t>(w * 32 + bit) | (flags << kFlagShift);
            }
            base += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) m.cnt[grp] = base;
    }
    // block total of live tiles
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) live += __shfl_down_sync(0xFFFFFFFFu, live, off);
    __shared__ long long warp_live[kCompactWarps];
    __shared__ bool is_last;
    if (lane == 0) warp_live[warp] = live;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long t = 0;
        for (int i = 0; i < kCompactWarps; ++i) t += warp_live[i];
        m.partial[blockIdx.x] = t;
        __threadfence();
        const unsigned int prev = atomicAdd(m.done, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---- last block: totals, stats, longest-first order
    __shared__ int hist[kOrderBuckets];
    __shared__ int warp_sum[kCompactWarps];
    __shared__ long long total_s;
    const int nb = (g.Tk + 1 < kOrderBuckets) ? (g.Tk + 1) : kOrderBuckets;   // count buckets
    const int64_t span = static_cast<int64_t>(g.Tk) + 1;
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
    if (warp == 0) {
        long long t = 0;
        for (unsigned int i = lane; i < gridDim.x; i += 32) t += __ldcg(&m.partial[i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t += __shfl_down_sync(0xFFFFFFFFu, t, off);
        if (lane == 0) total_s = t;
    }
    __syncthreads();
    // bucket of a count c in [0, Tk]; clamped so that no count can index past the histogram
    auto bucket = [&](int c) {
        const int64_t k = (static_cast<int64_t>(c < 0 ? 0 : c) * nb) / span;
        return static_cast<int>(k < nb - 1 ? k : nb - 1);
    };
    for (int i = threadIdx.x; i < g.G; i += blockDim.x) atomicAdd(&hist[bucket(__ldcg(&m.cnt[i]))], 1);
    __syncthreads();
    // exclusive scan of the histogram in descending bucket order (largest counts first)
    {
        constexpr int kPer = kOrderBuckets / kCompactThreads;
        int local[kPer];
        int sum = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int k = threadIdx.x * kPer + u;
            local[u] = (k < nb) ? hist[nb - 1 - k] : 0;
            sum += local[u];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += warp_sum[w];
        int run = before + incl - sum;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int k = threadIdx.x * kPer + u;
            if (k < nb) hist[nb - 1 - k] = run;
            run += local[u];
        }
    }
    if (threadIdx.x == 0) {
        const long long live_out = total_s;
        const long long live_in = step_mode ? live_in_src->live : 0;
        m.stats->live = live_out;
        m.stats->live_in = live_in;
        m.stats->newly_dead = step_mode ? (live_in - live_out) : 0;
        m.stats->last_step = step_mode ? step : -1;
        if (step_mode && plan) {
            plan->cum_qk += static_cast<unsigned long long>(live_in);
            plan->cum_pv += static_cast<unsigned long long>(live_out);
            plan->steps += 1ull;
        }
        *m.done = 0u;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < g.G; i += blockDim.x) {
        const int pos = atomicAdd(&hist[bucket(__ldcg(&m.cnt[i]))], 1);
        m.order[g.head_major ? i : pos] = i;
    }
}

// Divergence of two masks of one plan: out[0] += tiles live in a and not in b,
// out[1] += tiles live in b and not in a, over the R*W words of both bitmasks
// (bits >= Tk are 0 in every mask, so no word needs masking).  Grid-stride
// over words, a warp reduction, two atomics per warp; memory-bound.
__global__ void mask_diff_kernel(const uint32_t *a, const uint32_t *b, int64_t nwords, unsigned long long *out) {
    unsigned long long ca = 0, cb = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords; i += stride) {
        const uint32_t x = __ldg(a + i), y = __ldg(b + i);
        ca += static_cast<unsigned long long>(__popc(x & ~y));
        cb += static_cast<unsigned long long>(__popc(y & ~x));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ca += __shfl_down_sync(0xFFFFFFFFu, ca, o);
        cb += __shfl_down_sync(0xFFFFFFFFu, cb, o);
    }
    if ((threadIdx.x & 31) == 0 && (ca | cb)) {
        atomicAdd(out, ca);
        atomicAdd(out + 1, cb);
    }
}

}  // namespace lite
