// liteattn_internal.cuh -- device-side data structures shared by the
// LiteAttention kernels and the host library.
#pragma once

#include <cstdint>

namespace lite {

// Upper bound on key tiles per mask row handled by the attention kernel's
// shared-memory bitmap (W <= kMaxWords words): N <= 2^20 with 64-wide tiles.
constexpr int kMaxTk = 16384;
constexpr int kMaxWords = kMaxTk / 32;
constexpr int kMaxN = 1 << 20;

// Device status word values (mirror LITE_OK / LITE_ERR_DEVICE_TIMEOUT / LITE_ERR_DEVICE_CHECK).
constexpr int32_t kStatusOk = 0;
constexpr int32_t kStatusTimeout = -6;
constexpr int32_t kStatusCheck = -7;   // debug builds: a work item failed its checks

// Bounded-wait limit for every spin in the kernels (nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Shape of a plan, as the kernels see it.
struct Geometry {
    int B, H, N, d, Br, Bc;
    int Tq, Tk, W;     // query tiles, key tiles, 32-bit words per mask row
    int Gp, G;         // query-tile pairs per head, pairs in total
    int64_t R;         // mask rows = B*H*Tq
    int layout;        // 0: tensors [B][H][N][d]; 1: [B][N][H][d]
    int Ht;            // heads in the tensors (>= H: the plan covers H of them, from the pointer it is given)
    // Variable-length batches (seq_len != nullptr): sequence b has seq_len[b] <= N tokens at
    // token offset seq_off[b] of packed [total][H][d] tensors; the tile geometry above is that
    // of the longest sequence (N), and a shorter sequence's missing tiles are dead.
    const int32_t *seq_len;   // device [B] or nullptr
    const int64_t *seq_off;   // device [B] or nullptr
    int64_t tiles_total;      // valid (query tile, key tile) pairs: B*H*Tq*Tk, or the sum over sequences
    int64_t tokens;           // tokens per head in the tensors: B*N, or the sum of the lengths
    int head_major;           // work order: 1 = pairs in index (head-by-head) order, 0 = longest first
    int pair_stride;          // query tiles of a pair are pair_stride apart (1: adjacent; see pair_tiles)
};

// The two query tiles of pair p of one (batch, head), the second -1 when there is
// none.  The Tq tiles go in blocks of 2s (s = pair_stride): within a block, tile
// r pairs with tile r + s; a last, shorter block of m tiles pairs r with r +
// ceil(m/2).  With s = 1 pair p is tiles (2p, 2p + 1).  Every tile belongs to
// exactly one pair and there are ceil(Tq / 2) pairs.  A stride of one video frame
// (in tiles) pairs each query tile with the one a frame later, whose live key
// tiles overlap its own more than its neighbour's along the scan line do.
__host__ __device__ __forceinline__ void pair_tiles(int p, int Tq, int s, int &qa, int &qb) {
    const int full = Tq / (2 * s);           // complete blocks of 2s tiles
    if (p < full * s) {
        qa = (p / s) * 2 * s + p % s;
        qb = qa + s;
    } else {
        const int base = 2 * s * full, m = Tq - base, h = (m + 1) / 2, r = p - full * s;
        qa = base + r;
        qb = (r + h < m) ? qa + h : -1;
    }
}

// One head's K and V above this many bytes (a quarter of the 126 MB L2): run the
// pairs head by head so that each head's K and V stay in L2 while its pairs run,
// instead of longest first (which mixes heads and balances the grid's tail).
constexpr double kHeadMajorKVBytes = 32e6;

// Length of sequence b of a plan (N for fixed-length plans).
__device__ __forceinline__ int seq_length(const Geometry &g, int b) { return g.seq_len ? g.seq_len[b] : g.N; }

// Per-mask statistics block (device memory, written by the mask kernels).
struct MaskStats {
    int64_t live;         // live tiles in the mask
    int64_t live_in;      // live tiles of the incoming mask of the step that wrote it
    int64_t newly_dead;   // tiles killed in that step
    int32_t last_step;    // step index, -1 after reset/import
    int32_t pad;
};

// Accumulators of one output comparison (zeroed before each comparison).
struct ErrAcc {
    double sum_diff;        // sum |o - o_ref|
    double sum_ref;         // sum |o_ref|
    unsigned int max_bits;  // bits of max |o - o_ref| (non-negative floats order like unsigned ints)
    unsigned int pad;
};

// Per-plan device block: sticky status and plan-wide counters.
struct PlanDev {
    int32_t status;
    int32_t pad;
    unsigned long long cum_qk;
    unsigned long long cum_pv;
    unsigned long long steps;
    unsigned long long diff[2];   // mask comparison counters (lite_attn_mask_compare)
    ErrAcc err;                   // output comparison accumulators (lite_attn_output_error)
};

// Device views of one mask object.
struct MaskDev {
    uint32_t *bits;        // [R][W]
    uint32_t *list;        // [G][Tk] entries j | flags << 30, ascending j
    int32_t *cnt;          // [G]
    int32_t *order;        // [G] work order, descending count
    long long *partial;    // [compaction blocks] per-block live counts (scratch)
    unsigned int *done;    // compaction blocks finished (scratch, returns to 0)
    MaskStats *stats;
};

constexpr uint32_t kEntryMask = 0x3FFFFFFFu;
constexpr int kFlagShift = 30;

}  // namespace lite
