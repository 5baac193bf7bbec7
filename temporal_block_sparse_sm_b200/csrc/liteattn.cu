// liteattn.cu -- host side of the LiteAttention C ABI (include/liteattn.h):
// plans, skip-mask objects, argument checks, tensor-map encoding and the
// launches of the sm_100a kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "liteattn.h"
#include "attn_kernel.cuh"
#include "liteattn_internal.cuh"
#include "mask_kernels.cuh"
#include "metric_kernels.cuh"

using namespace lite;

namespace {

constexpr uint32_t kPlanMagic = 0x4C415050u;  // "LAPP"
constexpr uint32_t kMaskMagic = 0x4C414D4Bu;  // "LAMK"

std::atomic<int64_t> g_launches{0};

// NVTX range for the duration of a scope: the host side of each call shows up
// on profiler timelines (header-only NVTX3; a no-op without a tool attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Makes a plan's device current for the duration of a call and gives the caller
// back its own current device on exit, so a plan works whichever device the
// calling thread has selected (kernels, copies, events and synchronisation all
// go to the device that owns the plan's memory).
struct DeviceScope {
    int prev = -1;
    bool ok = false;
    explicit DeviceScope(int device) {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            cudaGetLastError();
            prev = -1;
            return;
        }
        ok = prev == device || cudaSetDevice(device) == cudaSuccess;
    }
    ~DeviceScope() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
    DeviceScope(const DeviceScope &) = delete;
    DeviceScope &operator=(const DeviceScope &) = delete;
};

constexpr int kMaxDevices = 64;

// Fault injection for tests: LITE_ATTN_FAULT=alloc|launch|status makes the
// matching host path report its error without touching the GPU;
// LITE_ATTN_FAULT=device_wait makes the attention kernel's first CTA wait on a
// barrier that nothing arrives on, so its bounded wait runs out and the step
// reports LITE_ERR_DEVICE_TIMEOUT through the status word.
bool fault(const char *what) {
    const char *e = std::getenv("LITE_ATTN_FAULT");
    return e && std::strcmp(e, what) == 0;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using AddrRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

struct DriverFns {
    EncodeTiledFn encode = nullptr;
    AddrRangeFn addr_range = nullptr;
    bool ok = false;
};

const DriverFns &driver() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q1, q2;
        void *p1 = nullptr, *p2 = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess)
            fns.encode = reinterpret_cast<EncodeTiledFn>(p1);
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess)
            fns.addr_range = reinterpret_cast<AddrRangeFn>(p2);
        fns.ok = fns.encode && fns.addr_range;
    });
    return fns;
}

struct TimingRec {
    cudaEvent_t a0, a1, s0, s1;
};

// Scratch of lite_attn_compact_noalloc: one fixed array per device that loads
// the library (held until exit).  Sized for LITE_NOALLOC_MAX_PAIRS pairs.
constexpr int kNoAllocMaxBlocks = LITE_NOALLOC_MAX_PAIRS / kCompactWarps;
struct NoAllocScratch {
    long long partial[kNoAllocMaxBlocks];
    unsigned int done;
    unsigned int pad;
    MaskStats stats;
};
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoAllocScratch)];

std::mutex g_noalloc_mu;
NoAllocScratch *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per
// device, with that device current).  In host code the symbol itself is only a
// host-side stand-in, so the kernel must be given this address.
NoAllocScratch *noalloc_scratch(int device) {
    if (device < 0 || device >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[device]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_noalloc_ptr[device] = static_cast<NoAllocScratch *>(ptr);
    }
    return g_noalloc_ptr[device];
}

}  // namespace

struct lite_attn_plan {
    uint32_t magic;
    Geometry g;
    int T;
    std::vector<float> taus;        // the per-step schedule: thresholds tau, or recall targets p
    int predicate = LITE_PRED_THRESHOLD;
    int device;
    PlanDev *dev;  // device block
    bool timing;
    std::vector<TimingRec> recs;
    std::vector<cudaEvent_t> pool;
    std::vector<int32_t> seq_lens;  // variable-length batches: host copy of the lengths (empty otherwise)
    void *seq_dev = nullptr;        // device lengths [B] (int32) then offsets [B] (int64)
    int64_t total_tokens = 0;       // tokens per head in the tensors' token dimension
    double dense_flops = 0.0;       // 4 * H * sum over sequences of N_b^2 * d
    cudaEvent_t done_ev = nullptr;  // recorded after each step's last kernel on the step's stream
    cudaStream_t aux = nullptr;     // non-blocking stream for the statistics' read-back
};

struct lite_attn_mask {
    uint32_t magic;
    lite_attn_plan *plan;
    int device;     // the plan's device (kept here so that destroy never reads the plan)
    void *mem;
    MaskDev d;
    int compact_blocks;
    cudaEvent_t done_ev = nullptr;  // recorded after the last work that wrote this mask, on its stream
};

namespace {

int cuda_err(cudaError_t e) { return e == cudaSuccess ? LITE_OK : LITE_ERR_CUDA; }

bool valid_plan(const lite_attn_plan *p) { return p && p->magic == kPlanMagic; }
bool valid_mask(const lite_attn_mask *m) { return m && m->magic == kMaskMagic; }

// Checks that [ptr, ptr + bytes) is device memory of `device` inside one allocation,
// and that ptr is aligned to `align` bytes (a power of two).
bool device_range_ok(const void *ptr, size_t bytes, int device, uintptr_t align = 16) {
    if (!ptr || (reinterpret_cast<uintptr_t>(ptr) & (align - 1u))) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return false;
    if (attr.type == cudaMemoryTypeDevice && attr.device != device) return false;
    CUdeviceptr basep = 0;
    size_t size = 0;
    if (driver().addr_range(&basep, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return false;
    const uintptr_t b = static_cast<uintptr_t>(basep), x = reinterpret_cast<uintptr_t>(ptr);
    return x >= b && x - b + bytes <= size;
}

// Bytes from the plan's first element to one past its last one in a tensor of Ht heads.
size_t tensor_extent_bytes(const Geometry &g) {
    const size_t d = static_cast<size_t>(g.d), N = static_cast<size_t>(g.N), H = static_cast<size_t>(g.H),
                 Ht = static_cast<size_t>(g.Ht), B = static_cast<size_t>(g.B);
    const size_t elems = g.seq_len ? (static_cast<size_t>(g.tokens) - 1) * Ht * d + H * d
                         : g.layout == LITE_LAYOUT_BNHD ? ((B - 1) * N * Ht + (N - 1) * Ht + H) * d
                                                         : ((B - 1) * Ht + H) * N * d;
    return elems * 2u;
}

bool overlaps(const void *a, const void *b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

// q, k, v as 4-D bf16 tensor maps, box of 64 elements of d by `box_rows` tokens of
// one (batch, head), 128-byte swizzle:
//   [B][Ht][N][d]: dims (d, N, H, B), box (64, rows, 1, 1);
//   [B][N][Ht][d]: dims (d, H, N, B), box (64, 1, rows, 1).
// H is the plan's head count and Ht the tensors' (the strides use Ht, and `ptr`
// points at the plan's first head).  Rows past N read as zeros in both, never
// the next head's tokens.
bool encode_map(CUtensorMap *m, const void *ptr, const Geometry &g, int box_rows) {
    const cuuint64_t d = static_cast<cuuint64_t>(g.d), N = static_cast<cuuint64_t>(g.N),
                     H = static_cast<cuuint64_t>(g.H), B = static_cast<cuuint64_t>(g.B),
                     Ht = static_cast<cuuint64_t>(g.Ht);
    const cuuint32_t rows = static_cast<cuuint32_t>(box_rows);
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4];
    if (g.seq_len) {   // packed [tokens][Ht][d]: the batch coordinate is always 0
        const cuuint64_t T = static_cast<cuuint64_t>(g.tokens);
        const cuuint64_t dd[4] = {d, H, T, 1u}, ss[3] = {d * 2u, Ht * d * 2u, T * Ht * d * 2u};
        const cuuint32_t bb[4] = {64u, 1u, rows, 1u};
        std::memcpy(dims, dd, sizeof dims), std::memcpy(strides, ss, sizeof strides), std::memcpy(box, bb, sizeof box);
    } else if (g.layout == LITE_LAYOUT_BNHD) {
        const cuuint64_t dd[4] = {d, H, N, B}, ss[3] = {d * 2u, Ht * d * 2u, N * Ht * d * 2u};
        const cuuint32_t bb[4] = {64u, 1u, rows, 1u};
        std::memcpy(dims, dd, sizeof dims), std::memcpy(strides, ss, sizeof strides), std::memcpy(box, bb, sizeof box);
    } else {
        const cuuint64_t dd[4] = {d, N, H, B}, ss[3] = {d * 2u, N * d * 2u, Ht * N * d * 2u};
        const cuuint32_t bb[4] = {64u, rows, 1u, 1u};
        std::memcpy(dims, dd, sizeof dims), std::memcpy(strides, ss, sizeof strides), std::memcpy(box, bb, sizeof box);
    }
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return driver().encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `param` is the step's threshold tau (QK-Skip plans) or recall target p (fixed-recall plans).
template <int D, int BR, int BC, bool RECALL>
int launch_attention(const lite_attn_plan *pl, const void *q, const void *k, const void *v, void *o,
                     const lite_attn_mask *min, lite_attn_mask *mout, float param, cudaStream_t stream) {
    using C = AttnCfg<D, BR, BC>;
    // the dynamic shared-memory limit is raised once per device (the plan's device is current here)
    static std::atomic<bool> attr_set[kMaxDevices];
    static std::mutex attr_mu;
    if (pl->device < 0 || pl->device >= kMaxDevices) return LITE_ERR_CUDA;
    if (!attr_set[pl->device].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(attr_mu);
        if (!attr_set[pl->device].load(std::memory_order_relaxed)) {
            if (cudaFuncSetAttribute(lite_attn_fwd_kernel<D, BR, BC, RECALL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(C::SMEM_BYTES)) != cudaSuccess) {
                cudaGetLastError();
                return LITE_ERR_CUDA;
            }
            attr_set[pl->device].store(true, std::memory_order_release);
        }
    }
    const Geometry &g = pl->g;
    CUtensorMap tq, tk, tv;
    if (!encode_map(&tq, q, g, 128) || !encode_map(&tk, k, g, BC) || !encode_map(&tv, v, g, BC))
        return LITE_ERR_CUDA;
    AttnParams p;
    p.list = min->d.list;
    p.cnt = min->d.cnt;
    p.order = min->d.order;
    p.bits_out = mout->d.bits;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.status = &pl->dev->status;
    p.probe_wait = fault("device_wait") ? 1 : 0;
    p.seq_len = g.seq_len;
    p.seq_off = g.seq_off;
    p.N = g.N;
    p.Tq = g.Tq;
    p.Tk = g.Tk;
    p.W = g.W;
    p.Gp = g.Gp;
    p.H = g.H;
    p.Ht = g.Ht;
    p.bnhd = g.layout == LITE_LAYOUT_BNHD ? 1 : 0;
    p.pair_stride = g.pair_stride;
    const double scale = 1.0 / std::sqrt(static_cast<double>(g.d));
    p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
    if (RECALL) {
        p.thr_raw = -INFINITY;
        p.recall_c = static_cast<float>((1.0 - static_cast<double>(param)) / static_cast<double>(param));
    } else {
        p.thr_raw = std::isinf(param) ? -INFINITY : static_cast<float>(static_cast<double>(param) / scale);
        p.recall_c = 0.0f;
    }
    lite_attn_fwd_kernel<D, BR, BC, RECALL><<<g.G, C::NTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
    g_launches.fetch_add(1);
    return cuda_err(cudaGetLastError());
}

int launch_compact(const lite_attn_plan *pl, lite_attn_mask *m, int step_mode, const MaskStats *live_in_src,
                   int step, cudaStream_t stream) {
    mask_compact_kernel<<<m->compact_blocks, kCompactThreads, 0, stream>>>(m->d, pl->g, step_mode, live_in_src, step,
                                                                           pl->dev);
    g_launches.fetch_add(1);
    return cuda_err(cudaGetLastError());
}

int launch_reset(const lite_attn_plan *pl, lite_attn_mask *m, cudaStream_t stream) {
    const Geometry &g = pl->g;
    int64_t work = std::max<int64_t>(g.R * g.W, static_cast<int64_t>(g.G) * g.Tk);
    int blocks = static_cast<int>(std::min<int64_t>((work + 255) / 256, 148 * 16));
    if (blocks < 1) blocks = 1;
    mask_reset_kernel<<<blocks, 256, 0, stream>>>(m->d, g);
    g_launches.fetch_add(1);
    return cuda_err(cudaGetLastError());
}

cudaEvent_t take_event(lite_attn_plan *pl) {
    if (!pl->pool.empty()) {
        cudaEvent_t e = pl->pool.back();
        pl->pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void recycle_records(lite_attn_plan *pl) {
    for (auto &r : pl->recs) {
        pl->pool.push_back(r.a0);
        pl->pool.push_back(r.a1);
        pl->pool.push_back(r.s0);
        pl->pool.push_back(r.s1);
    }
    pl->recs.clear();
}


// Plan creation shared by the fixed-length and variable-length entry points
// (seq_lens: host [B] lengths, or nullptr for B sequences of N tokens).
// schedule: per-step thresholds tau (predicate LITE_PRED_THRESHOLD) or recall targets p
// (LITE_PRED_RECALL).
int create_plan(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc, const float *schedule,
                int T, int layout, int heads_total, const int32_t *seq_lens, int predicate = LITE_PRED_THRESHOLD,
                int pair_stride = 1) {
    if (!out) return LITE_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || H < 1 || T < 1 || !schedule) return LITE_ERR_INVALID_ARG;
    if (pair_stride == 0) pair_stride = 1;
    if (pair_stride < 1) return LITE_ERR_INVALID_ARG;
    if (layout != LITE_LAYOUT_BHND && layout != LITE_LAYOUT_BNHD) return LITE_ERR_INVALID_ARG;
    if (predicate != LITE_PRED_THRESHOLD && predicate != LITE_PRED_RECALL) return LITE_ERR_INVALID_ARG;
    if (heads_total == 0) heads_total = H;
    if (heads_total < H) return LITE_ERR_INVALID_ARG;
    if (d < 1 || Br < 1 || Bc < 1) return LITE_ERR_INVALID_ARG;
    for (int t = 0; t < T; ++t) {
        const float x = schedule[t];
        if (predicate == LITE_PRED_THRESHOLD && (std::isnan(x) || x > 0.0f)) return LITE_ERR_INVALID_ARG;
        if (predicate == LITE_PRED_RECALL && !(x > 0.0f && x <= 1.0f)) return LITE_ERR_INVALID_ARG;
    }
    const bool cfg_ok = (d == 64 && Br == 64 && Bc == 64) || (d == 128 && Br == 128 && Bc == 128);
    if (!cfg_ok || N < 1 || N > kMaxN) return LITE_ERR_UNSUPPORTED;
    // a pair stride needs one query tile per 128-row slot, and one tile geometry for the batch
    if (pair_stride > 1 && (Br != 128 || seq_lens)) return LITE_ERR_UNSUPPORTED;
    int64_t total = static_cast<int64_t>(B) * N;   // tokens per head over the batch
    if (seq_lens) {
        total = 0;
        for (int b = 0; b < B; ++b) total += seq_lens[b];
        if (total >= (int64_t(1) << 31)) return LITE_ERR_UNSUPPORTED;
    }
    if (total * heads_total * d > (int64_t(1) << 40)) return LITE_ERR_UNSUPPORTED;
    if (fault("alloc")) return LITE_ERR_ALLOC;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LITE_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LITE_ERR_CUDA;
    if (prop.major != 10) return LITE_ERR_CUDA;
    if (!driver().ok) return LITE_ERR_CUDA;
    Geometry g;
    g.B = B;
    g.H = H;
    g.N = N;
    g.d = d;
    g.Br = Br;
    g.Bc = Bc;
    g.Tq = (N + Br - 1) / Br;
    g.Tk = (N + Bc - 1) / Bc;
    g.W = (g.Tk + 31) / 32;
    g.Gp = (g.Tq + 1) / 2;
    const int64_t G = static_cast<int64_t>(B) * H * g.Gp;
    if (G > (int64_t(1) << 30)) return LITE_ERR_UNSUPPORTED;
    g.G = static_cast<int>(G);
    g.R = static_cast<int64_t>(B) * H * g.Tq;
    g.layout = layout;
    g.Ht = heads_total;
    g.pair_stride = pair_stride;
    g.seq_len = nullptr;
    g.seq_off = nullptr;
    g.tokens = total;
    g.head_major = (4.0 * N * d > kHeadMajorKVBytes) ? 1 : 0;   // K + V of the longest sequence, bf16
    lite_attn_plan *pl = new (std::nothrow) lite_attn_plan();
    if (!pl) return LITE_ERR_ALLOC;
    pl->T = T;
    pl->taus.assign(schedule, schedule + T);
    pl->predicate = predicate;
    pl->device = dev;
    pl->dev = nullptr;
    pl->timing = false;
    pl->total_tokens = total;
    if (seq_lens) {
        pl->seq_lens.assign(seq_lens, seq_lens + B);
        std::vector<int64_t> off(B);
        int64_t acc = 0, tiles = 0;
        double flops = 0.0;
        for (int b = 0; b < B; ++b) {
            off[b] = acc;
            acc += seq_lens[b];
            const int64_t tq = (seq_lens[b] + Br - 1) / Br, tk = (seq_lens[b] + Bc - 1) / Bc;
            tiles += static_cast<int64_t>(H) * tq * tk;
            flops += 4.0 * H * static_cast<double>(seq_lens[b]) * seq_lens[b] * d;
        }
        g.tiles_total = tiles;
        pl->dense_flops = flops;
        const size_t bytes = static_cast<size_t>(B) * (sizeof(int32_t) + sizeof(int64_t)) + 8;
        if (cudaMalloc(&pl->seq_dev, bytes) != cudaSuccess) {
            cudaGetLastError();
            delete pl;
            return LITE_ERR_ALLOC;
        }
        int64_t *d_off = reinterpret_cast<int64_t *>(pl->seq_dev);                  // 8-byte aligned first
        int32_t *d_len = reinterpret_cast<int32_t *>(d_off + B);
        if (cudaMemcpy(d_off, off.data(), B * sizeof(int64_t), cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMemcpy(d_len, seq_lens, B * sizeof(int32_t), cudaMemcpyHostToDevice) != cudaSuccess) {
            cudaFree(pl->seq_dev);
            delete pl;
            return LITE_ERR_CUDA;
        }
        g.seq_off = d_off;
        g.seq_len = d_len;
    } else {
        g.tiles_total = g.R * g.Tk;
        pl->dense_flops = 4.0 * B * H * static_cast<double>(N) * N * d;
    }
    pl->g = g;
    if (cudaMalloc(&pl->dev, sizeof(PlanDev)) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(pl->seq_dev);
        delete pl;
        return LITE_ERR_ALLOC;
    }
    if (cudaMemset(pl->dev, 0, sizeof(PlanDev)) != cudaSuccess) {
        cudaFree(pl->dev);
        cudaFree(pl->seq_dev);
        delete pl;
        return LITE_ERR_CUDA;
    }
    if (cudaEventCreateWithFlags(&pl->done_ev, cudaEventDisableTiming) != cudaSuccess ||
        cudaStreamCreateWithFlags(&pl->aux, cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();
        if (pl->done_ev) cudaEventDestroy(pl->done_ev);
        cudaFree(pl->dev);
        cudaFree(pl->seq_dev);
        delete pl;
        return LITE_ERR_CUDA;
    }
    pl->magic = kPlanMagic;
    *out = pl;
    return LITE_OK;
}

#ifdef LITE_DEBUG_CHECKS
// Checked builds only: the softmax's two exponential paths, the FMA-pipe
// polynomial (ptx::exp2_poly2) and MUFU ex2 (ptx::ex2), on caller inputs, so a
// test can hold them against exact 2^x.  Grid-stride over pairs.
__global__ void exp2_paths_kernel(const float *x, float *y_poly, float *y_mufu, int64_t n) {
    const int64_t stride = 2 * static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n; i += stride) {
        const bool two = i + 1 < n;
        const float a = x[i], b = two ? x[i + 1] : 0.0f;
        float p0, p1;
        ptx::exp2_poly2(a, b, p0, p1);
        y_poly[i] = p0;
        y_mufu[i] = ptx::ex2(a);
        if (two) {
            y_poly[i + 1] = p1;
            y_mufu[i + 1] = ptx::ex2(b);
        }
    }
}
#endif

}  // namespace

extern "C" {

const char *lite_attn_error_string(int code) {
    switch (code) {
        case LITE_OK: return "ok";
        case LITE_ERR_INVALID_ARG: return "invalid argument";
        case LITE_ERR_UNSUPPORTED: return "unsupported shape or tile configuration";
        case LITE_ERR_PLAN_MISMATCH: return "mask does not belong to this plan";
        case LITE_ERR_ALLOC: return "allocation failed";
        case LITE_ERR_CUDA: return "CUDA error";
        case LITE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case LITE_ERR_DEVICE_CHECK: return "device-side check failed (debug build)";
        default: return "unknown error";
    }
}

int64_t lite_attn_launch_count(void) { return g_launches.load(); }

int lite_attn_plan_create(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                          const float *threshold_schedule, int T) {
    return lite_attn_plan_create_ex(out, B, H, N, d, Br, Bc, threshold_schedule, T, LITE_LAYOUT_BHND, 0);
}

int lite_attn_plan_create_ex(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                             const float *threshold_schedule, int T, int layout, int heads_total) {
    return create_plan(out, B, H, N, d, Br, Bc, threshold_schedule, T, layout, heads_total, nullptr);
}

int lite_attn_plan_create_recall(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                                 const float *recall_schedule, int T, int layout, int heads_total) {
    return create_plan(out, B, H, N, d, Br, Bc, recall_schedule, T, layout, heads_total, nullptr, LITE_PRED_RECALL);
}

int lite_attn_plan_create_opts(lite_attn_plan_t *out, int B, int H, int N, int d, int Br, int Bc,
                               const float *schedule, int T, const lite_attn_plan_options_t *opts) {
    if (!out) return LITE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!opts) return LITE_ERR_INVALID_ARG;
    return create_plan(out, B, H, N, d, Br, Bc, schedule, T, opts->layout, opts->heads_total, nullptr,
                       opts->predicate, opts->pair_stride);
}

int lite_attn_plan_predicate(lite_attn_plan_t plan, int *predicate) {
    if (!valid_plan(plan) || !predicate) return LITE_ERR_INVALID_ARG;
    *predicate = plan->predicate;
    return LITE_OK;
}

int lite_attn_plan_create_varlen(lite_attn_plan_t *out, int B, int H, const int32_t *seq_lens, int d, int Br,
                                 int Bc, const float *threshold_schedule, int T) {
    if (!out) return LITE_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || !seq_lens) return LITE_ERR_INVALID_ARG;
    int N = 0;
    for (int b = 0; b < B; ++b) {
        if (seq_lens[b] < 1) return LITE_ERR_INVALID_ARG;
        N = std::max(N, static_cast<int>(seq_lens[b]));
    }
    return create_plan(out, B, H, N, d, Br, Bc, threshold_schedule, T, LITE_LAYOUT_BNHD, 0, seq_lens);
}

int lite_attn_plan_destroy(lite_attn_plan_t plan) {
    if (!plan) return LITE_OK;
    if (!valid_plan(plan)) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(plan->device);
    cudaDeviceSynchronize();
    recycle_records(plan);
    for (cudaEvent_t e : plan->pool) cudaEventDestroy(e);
    cudaEventDestroy(plan->done_ev);
    cudaStreamDestroy(plan->aux);
    cudaFree(plan->dev);
    if (plan->seq_dev) cudaFree(plan->seq_dev);
    plan->magic = 0;
    delete plan;
    return LITE_OK;
}

int lite_attn_plan_pair_tiles(lite_attn_plan_t plan, int pair, int *tile_a, int *tile_b) {
    if (!valid_plan(plan) || !tile_a || !tile_b || pair < 0 || pair >= plan->g.Gp) return LITE_ERR_INVALID_ARG;
    pair_tiles(pair, plan->g.Tq, plan->g.pair_stride, *tile_a, *tile_b);
    return LITE_OK;
}

int lite_attn_plan_info(lite_attn_plan_t plan, int *Tq, int *Tk, int *W, int *G) {
    if (!valid_plan(plan)) return LITE_ERR_INVALID_ARG;
    if (Tq) *Tq = plan->g.Tq;
    if (Tk) *Tk = plan->g.Tk;
    if (W) *W = plan->g.W;
    if (G) *G = plan->g.G;
    return LITE_OK;
}

int lite_attn_mask_create(lite_attn_plan_t plan, lite_attn_mask_t *out) {
    if (!out) return LITE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!valid_plan(plan)) return LITE_ERR_INVALID_ARG;
    if (fault("alloc")) return LITE_ERR_ALLOC;
    const Geometry &g = plan->g;
    const int blocks = (g.G + kCompactWarps - 1) / kCompactWarps;
    auto align = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t sz_bits = align(static_cast<size_t>(g.R) * g.W * 4);
    const size_t sz_list = align(static_cast<size_t>(g.G) * g.Tk * 4);
    const size_t sz_cnt = align(static_cast<size_t>(g.G) * 4);
    const size_t sz_part = align(static_cast<size_t>(blocks) * 8);
    const size_t sz_done = 256;
    const size_t sz_stats = align(sizeof(MaskStats));
    const size_t total = sz_bits + sz_list + 2 * sz_cnt + sz_part + sz_done + sz_stats;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    lite_attn_mask *m = new (std::nothrow) lite_attn_mask();
    if (!m) return LITE_ERR_ALLOC;
    if (cudaMalloc(&m->mem, total) != cudaSuccess) {
        cudaGetLastError();
        delete m;
        return LITE_ERR_ALLOC;
    }
    uint8_t *b = static_cast<uint8_t *>(m->mem);
    m->d.bits = reinterpret_cast<uint32_t *>(b);
    b += sz_bits;
    m->d.list = reinterpret_cast<uint32_t *>(b);
    b += sz_list;
    m->d.cnt = reinterpret_cast<int32_t *>(b);
    b += sz_cnt;
    m->d.order = reinterpret_cast<int32_t *>(b);
    b += sz_cnt;
    m->d.partial = reinterpret_cast<long long *>(b);
    b += sz_part;
    m->d.done = reinterpret_cast<unsigned int *>(b);
    b += sz_done;
    m->d.stats = reinterpret_cast<MaskStats *>(b);
    m->plan = plan;
    m->device = plan->device;
    m->compact_blocks = blocks;
    int rc = cuda_err(cudaEventCreateWithFlags(&m->done_ev, cudaEventDisableTiming));
    if (rc == LITE_OK) rc = launch_reset(plan, m, nullptr);
    if (rc == LITE_OK) rc = cuda_err(cudaDeviceSynchronize());
    if (rc != LITE_OK) {
        cudaGetLastError();
        if (m->done_ev) cudaEventDestroy(m->done_ev);
        cudaFree(m->mem);
        delete m;
        return rc;
    }
    m->magic = kMaskMagic;
    *out = m;
    return LITE_OK;
}

int lite_attn_mask_destroy(lite_attn_mask_t mask) {
    if (!mask) return LITE_OK;
    if (!valid_mask(mask)) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(mask->device);
    cudaDeviceSynchronize();
    cudaEventDestroy(mask->done_ev);
    cudaFree(mask->mem);
    mask->magic = 0;
    delete mask;
    return LITE_OK;
}

int lite_attn_mask_reset(lite_attn_mask_t mask, void *stream) {
    if (!valid_mask(mask)) return LITE_ERR_INVALID_ARG;
    NvtxRange range("lite_attn_mask_reset");
    if (fault("launch")) return LITE_ERR_CUDA;
    DeviceScope ds(mask->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    const int rc = launch_reset(mask->plan, mask, static_cast<cudaStream_t>(stream));
    if (rc != LITE_OK) return rc;
    return cuda_err(cudaEventRecord(mask->done_ev, static_cast<cudaStream_t>(stream)));
}

int lite_attn_mask_import(lite_attn_mask_t mask, const uint32_t *host_bits, void *stream) {
    if (!valid_mask(mask) || !host_bits) return LITE_ERR_INVALID_ARG;
    NvtxRange range("lite_attn_mask_import");
    const Geometry &g = mask->plan->g;
    const auto &lens = mask->plan->seq_lens;
    for (int64_t r = 0; r < g.R; ++r) {
        // bits must name existing tiles: key tiles < Tk of the row's sequence, and no bits at
        // all in rows of query tiles the sequence does not have
        const int Nb = lens.empty() ? g.N : lens[static_cast<size_t>((r / g.Tq) / g.H)];
        const int Tqb = (Nb + g.Br - 1) / g.Br, Tkb = (Nb + g.Bc - 1) / g.Bc;
        const bool row_exists = (r % g.Tq) < Tqb;
        for (int w = 0; w < g.W; ++w) {
            const int nvalid = row_exists ? Tkb - 32 * w : 0;
            const uint32_t keep = nvalid >= 32 ? 0xFFFFFFFFu : nvalid <= 0 ? 0u : ((1u << nvalid) - 1u);
            if (host_bits[r * g.W + w] & ~keep) return LITE_ERR_INVALID_ARG;
        }
    }
    if (fault("launch")) return LITE_ERR_CUDA;
    DeviceScope ds(mask->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(g.R) * g.W * 4;
    int rc = cuda_err(cudaMemcpyAsync(mask->d.bits, host_bits, bytes, cudaMemcpyHostToDevice, s));
    if (rc != LITE_OK) return rc;
    // the caller may reuse host_bits on return
    rc = cuda_err(cudaStreamSynchronize(s));
    if (rc != LITE_OK) return rc;
    rc = launch_compact(mask->plan, mask, 0, nullptr, -1, s);
    if (rc != LITE_OK) return rc;
    return cuda_err(cudaEventRecord(mask->done_ev, s));
}

int lite_attn_mask_export(lite_attn_mask_t mask, uint32_t *host_bits, void *stream) {
    if (!valid_mask(mask) || !host_bits) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(mask->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    const Geometry &g = mask->plan->g;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(g.R) * g.W * 4;
    int rc = cuda_err(cudaMemcpyAsync(host_bits, mask->d.bits, bytes, cudaMemcpyDeviceToHost, s));
    if (rc != LITE_OK) return rc;
    return cuda_err(cudaStreamSynchronize(s));
}

int lite_attn_mask_export_lists(lite_attn_mask_t mask, uint32_t *host_list, int32_t *host_cnt, int32_t *host_order,
                                void *stream) {
    if (!valid_mask(mask)) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(mask->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    const Geometry &g = mask->plan->g;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc = LITE_OK;
    if (host_list && rc == LITE_OK)
        rc = cuda_err(cudaMemcpyAsync(host_list, mask->d.list, static_cast<size_t>(g.G) * g.Tk * 4,
                                      cudaMemcpyDeviceToHost, s));
    if (host_cnt && rc == LITE_OK)
        rc = cuda_err(cudaMemcpyAsync(host_cnt, mask->d.cnt, static_cast<size_t>(g.G) * 4, cudaMemcpyDeviceToHost, s));
    if (host_order && rc == LITE_OK)
        rc = cuda_err(
            cudaMemcpyAsync(host_order, mask->d.order, static_cast<size_t>(g.G) * 4, cudaMemcpyDeviceToHost, s));
    if (rc != LITE_OK) return rc;
    return cuda_err(cudaStreamSynchronize(s));
}

int lite_attn_step(lite_attn_plan_t plan, const void *q, const void *k, const void *v, void *o,
                   lite_attn_mask_t mask_in, lite_attn_mask_t mask_out, int step, void *stream) {
    if (!valid_plan(plan) || !valid_mask(mask_in) || !valid_mask(mask_out)) return LITE_ERR_INVALID_ARG;
    if (mask_in->plan != plan || mask_out->plan != plan) return LITE_ERR_PLAN_MISMATCH;
    if (step < 0 || step >= plan->T) return LITE_ERR_INVALID_ARG;
    const Geometry &g = plan->g;
    const size_t bytes = tensor_extent_bytes(g);
    if (!device_range_ok(q, bytes, plan->device) || !device_range_ok(k, bytes, plan->device) ||
        !device_range_ok(v, bytes, plan->device) || !device_range_ok(o, bytes, plan->device))
        return LITE_ERR_INVALID_ARG;
    if (overlaps(o, q, bytes) || overlaps(o, k, bytes) || overlaps(o, v, bytes)) return LITE_ERR_INVALID_ARG;
    if (fault("launch")) return LITE_ERR_CUDA;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const float param = plan->taus[step];
    const bool recall = plan->predicate == LITE_PRED_RECALL;
    TimingRec rec{};
    if (plan->timing) {
        rec.a0 = take_event(plan);
        rec.a1 = take_event(plan);
        rec.s0 = take_event(plan);
        rec.s1 = take_event(plan);
        if (!rec.a0 || !rec.a1 || !rec.s0 || !rec.s1) return LITE_ERR_CUDA;
        cudaEventRecord(rec.s0, s);
        cudaEventRecord(rec.a0, s);
    }
    NvtxRange range("lite_attn_step");
    int rc;
    {
        NvtxRange r("attention");
        if (g.d == 64)
            rc = recall ? launch_attention<64, 64, 64, true>(plan, q, k, v, o, mask_in, mask_out, param, s)
                        : launch_attention<64, 64, 64, false>(plan, q, k, v, o, mask_in, mask_out, param, s);
        else
            rc = recall ? launch_attention<128, 128, 128, true>(plan, q, k, v, o, mask_in, mask_out, param, s)
                        : launch_attention<128, 128, 128, false>(plan, q, k, v, o, mask_in, mask_out, param, s);
    }
    if (rc != LITE_OK) return rc;
    if (plan->timing) cudaEventRecord(rec.a1, s);
    {
        NvtxRange r("compaction");
        rc = launch_compact(plan, mask_out, 1, mask_in->d.stats, step, s);
    }
    if (rc != LITE_OK) return rc;
    if (plan->timing) {
        cudaEventRecord(rec.s1, s);
        plan->recs.push_back(rec);
    }
    // what lite_attn_stats waits for: the step's kernels wrote the plan's counters,
    // mask_out's lists and statistics, and read mask_in
    rc = cuda_err(cudaEventRecord(plan->done_ev, s));
    if (rc == LITE_OK) rc = cuda_err(cudaEventRecord(mask_out->done_ev, s));
    if (rc == LITE_OK && mask_in != mask_out) rc = cuda_err(cudaEventRecord(mask_in->done_ev, s));
    return rc;
}

int lite_attn_stats(lite_attn_plan_t plan, lite_attn_mask_t mask, lite_attn_stats_t *out) {
    if (!valid_plan(plan) || !valid_mask(mask) || !out) return LITE_ERR_INVALID_ARG;
    if (mask->plan != plan) return LITE_ERR_PLAN_MISMATCH;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    // Wait only for the work that wrote these counters (the plan's last step, the
    // mask's last writer), then read them back on the plan's own non-blocking
    // stream: other streams of the device keep running.
    int rc = cuda_err(cudaEventSynchronize(plan->done_ev));
    if (rc == LITE_OK) rc = cuda_err(cudaEventSynchronize(mask->done_ev));
    if (rc != LITE_OK) return rc;
    MaskStats ms;
    PlanDev pd;
    rc = cuda_err(cudaMemcpyAsync(&ms, mask->d.stats, sizeof ms, cudaMemcpyDeviceToHost, plan->aux));
    if (rc == LITE_OK) rc = cuda_err(cudaMemcpyAsync(&pd, plan->dev, sizeof pd, cudaMemcpyDeviceToHost, plan->aux));
    if (rc == LITE_OK) rc = cuda_err(cudaStreamSynchronize(plan->aux));
    if (rc != LITE_OK) return rc;
    const Geometry &g = plan->g;
    std::memset(out, 0, sizeof *out);
    out->tiles_total = g.tiles_total;
    out->live_out = ms.live;
    out->live_in = ms.live_in;
    out->qk_tiles = ms.live_in;
    out->pv_tiles = ms.last_step >= 0 ? ms.live : 0;
    out->newly_dead = ms.newly_dead;
    out->skip_fraction = out->tiles_total ? 1.0 - static_cast<double>(ms.live) / out->tiles_total : 0.0;
    const double tile_flops = 2.0 * g.Br * g.Bc * g.d;
    out->executed_flops = tile_flops * static_cast<double>(out->qk_tiles + out->pv_tiles);
    out->dense_flops = plan->dense_flops;
    out->cum_qk_tiles = static_cast<int64_t>(pd.cum_qk);
    out->cum_pv_tiles = static_cast<int64_t>(pd.cum_pv);
    out->cum_steps = static_cast<int64_t>(pd.steps);
    out->device_status = fault("status") ? LITE_ERR_DEVICE_TIMEOUT : pd.status;
    out->last_step = ms.last_step;
    if (out->device_status == LITE_OK) return LITE_OK;
    return out->device_status == LITE_ERR_DEVICE_CHECK ? LITE_ERR_DEVICE_CHECK : LITE_ERR_DEVICE_TIMEOUT;
}

int lite_attn_mask_compare(lite_attn_mask_t a, lite_attn_mask_t b, int64_t *only_a, int64_t *only_b,
                           void *stream) {
    if (!valid_mask(a) || !valid_mask(b) || !only_a || !only_b) return LITE_ERR_INVALID_ARG;
    if (a->plan != b->plan) return LITE_ERR_PLAN_MISMATCH;
    if (fault("launch")) return LITE_ERR_CUDA;
    NvtxRange range("lite_attn_mask_compare");
    DeviceScope ds(a->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    lite_attn_plan *pl = a->plan;
    const Geometry &g = pl->g;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long *cnt = pl->dev->diff;
    int rc = cuda_err(cudaMemsetAsync(cnt, 0, 2 * sizeof(unsigned long long), s));
    if (rc != LITE_OK) return rc;
    const int64_t nwords = g.R * g.W;
    const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((nwords + 255) / 256, 148 * 8)));
    mask_diff_kernel<<<blocks, 256, 0, s>>>(a->d.bits, b->d.bits, nwords, cnt);
    g_launches.fetch_add(1);
    rc = cuda_err(cudaGetLastError());
    if (rc != LITE_OK) return rc;
    unsigned long long host[2] = {0, 0};
    rc = cuda_err(cudaMemcpyAsync(host, cnt, sizeof host, cudaMemcpyDeviceToHost, s));
    if (rc == LITE_OK) rc = cuda_err(cudaStreamSynchronize(s));
    if (rc != LITE_OK) return rc;
    *only_a = static_cast<int64_t>(host[0]);
    *only_b = static_cast<int64_t>(host[1]);
    return LITE_OK;
}

int lite_attn_output_error(lite_attn_plan_t plan, const void *o, const void *o_ref, double *out, void *stream) {
    if (!valid_plan(plan) || !out) return LITE_ERR_INVALID_ARG;
    const Geometry &g = plan->g;
    if (g.Ht != g.H) return LITE_ERR_INVALID_ARG;   // contiguous tensors only
    NvtxRange range("lite_attn_output_error");
    const size_t n = static_cast<size_t>(g.tokens) * g.H * g.d;
    if (!device_range_ok(o, n * 2u, plan->device) || !device_range_ok(o_ref, n * 2u, plan->device))
        return LITE_ERR_INVALID_ARG;
    if (fault("launch")) return LITE_ERR_CUDA;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ErrAcc *acc = &plan->dev->err;
    int rc = cuda_err(cudaMemsetAsync(acc, 0, sizeof(ErrAcc), s));
    if (rc != LITE_OK) return rc;
    const int64_t n8 = static_cast<int64_t>(n / 8);   // d is 64 or 128: n is a multiple of 8
    const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, 148 * 8)));
    output_error_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(o), static_cast<const uint4 *>(o_ref), n8,
                                               acc);
    g_launches.fetch_add(1);
    rc = cuda_err(cudaGetLastError());
    if (rc != LITE_OK) return rc;
    ErrAcc host;
    rc = cuda_err(cudaMemcpyAsync(&host, acc, sizeof host, cudaMemcpyDeviceToHost, s));
    if (rc == LITE_OK) rc = cuda_err(cudaStreamSynchronize(s));
    if (rc != LITE_OK) return rc;
    float mx;
    std::memcpy(&mx, &host.max_bits, sizeof mx);
    out[0] = host.sum_diff;
    out[1] = static_cast<double>(mx);
    out[2] = host.sum_ref;
    return LITE_OK;
}

int lite_attn_timing_enable(lite_attn_plan_t plan, int enable) {
    if (!valid_plan(plan)) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    cudaDeviceSynchronize();
    recycle_records(plan);
    plan->timing = enable != 0;
    return LITE_OK;
}

int lite_attn_timing_read(lite_attn_plan_t plan, double *attn_ms, double *step_ms, int64_t *n_steps) {
    if (!valid_plan(plan)) return LITE_ERR_INVALID_ARG;
    DeviceScope ds(plan->device);
    if (!ds.ok) return LITE_ERR_CUDA;
    double a = 0.0, s = 0.0;
    for (auto &r : plan->recs) {
        if (cudaEventSynchronize(r.s1) != cudaSuccess) return LITE_ERR_CUDA;
        float x = 0.f, y = 0.f;
        if (cudaEventElapsedTime(&x, r.a0, r.a1) != cudaSuccess) return LITE_ERR_CUDA;
        if (cudaEventElapsedTime(&y, r.s0, r.s1) != cudaSuccess) return LITE_ERR_CUDA;
        a += x;
        s += y;
    }
    if (attn_ms) *attn_ms = a;
    if (step_ms) *step_ms = s;
    if (n_steps) *n_steps = static_cast<int64_t>(plan->recs.size());
    recycle_records(plan);
    return LITE_OK;
}

int lite_attn_compact_noalloc(const uint32_t *bits, int B, int H, int N, int Br, int Bc, uint32_t *list,
                              int32_t *cnt, int32_t *order, int64_t *live_total, void *stream) {
    if (!bits || !list || !cnt || !order || !live_total || B < 1 || H < 1) return LITE_ERR_INVALID_ARG;
    const bool cfg_ok = (Br == 64 && Bc == 64) || (Br == 128 && Bc == 128);
    if (!cfg_ok || N < 1 || N > kMaxN) return LITE_ERR_UNSUPPORTED;
    Geometry g;
    g.B = B;
    g.H = H;
    g.N = N;
    g.d = Bc;
    g.Br = Br;
    g.Bc = Bc;
    g.Tq = (N + Br - 1) / Br;
    g.Tk = (N + Bc - 1) / Bc;
    g.W = (g.Tk + 31) / 32;
    g.Gp = (g.Tq + 1) / 2;
    const int64_t G = static_cast<int64_t>(B) * H * g.Gp;
    if (G > LITE_NOALLOC_MAX_PAIRS) return LITE_ERR_UNSUPPORTED;
    g.G = static_cast<int>(G);
    g.R = static_cast<int64_t>(B) * H * g.Tq;
    g.layout = LITE_LAYOUT_BHND;  // masks do not depend on the tensor layout
    g.Ht = H;
    g.pair_stride = 1;            // adjacent query tiles, the mask store's default pairing
    g.seq_len = nullptr;
    g.seq_off = nullptr;
    g.tiles_total = g.R * g.Tk;
    g.tokens = static_cast<int64_t>(B) * N;
    g.head_major = 0;   // the documented longest-first order
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LITE_ERR_CUDA;
    // Every buffer must be memory of the current device, inside one allocation,
    // large enough and aligned for its element type; the outputs must not overlap
    // the bitmask or one another.  Nothing is launched otherwise.
    const size_t b_bits = static_cast<size_t>(g.R) * g.W * 4, b_list = static_cast<size_t>(g.G) * g.Tk * 4,
                 b_cnt = static_cast<size_t>(g.G) * 4;
    if (!device_range_ok(bits, b_bits, dev, 4) || !device_range_ok(list, b_list, dev, 4) ||
        !device_range_ok(cnt, b_cnt, dev, 4) || !device_range_ok(order, b_cnt, dev, 4) ||
        !device_range_ok(live_total, sizeof(int64_t), dev, 8))
        return LITE_ERR_INVALID_ARG;
    auto disjoint = [](const void *a, size_t na, const void *b, size_t nb) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
        return x + na <= y || y + nb <= x;
    };
    const void *bufs[5] = {bits, list, cnt, order, live_total};
    const size_t lens[5] = {b_bits, b_list, b_cnt, b_cnt, sizeof(int64_t)};
    for (int i = 0; i < 5; ++i)
        for (int j = i + 1; j < 5; ++j)
            if (!disjoint(bufs[i], lens[i], bufs[j], lens[j])) return LITE_ERR_INVALID_ARG;
    if (stream) {   // the stream must belong to the current device
        int sdev = -1;
        if (cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) != cudaSuccess) {
            cudaGetLastError();
            return LITE_ERR_INVALID_ARG;
        }
        if (sdev != dev) return LITE_ERR_INVALID_ARG;
    }
    NoAllocScratch *scr = noalloc_scratch(dev);
    if (!scr) return LITE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the completion counter must start at zero (the kernel's last block also resets it)
    int rc = cuda_err(cudaMemsetAsync(&scr->done, 0, sizeof(unsigned int), s));
    if (rc != LITE_OK) return rc;
    MaskDev m;
    m.bits = const_cast<uint32_t *>(bits);
    m.list = list;
    m.cnt = cnt;
    m.order = order;
    m.partial = scr->partial;
    m.done = &scr->done;
    m.stats = &scr->stats;
    const int blocks = (g.G + kCompactWarps - 1) / kCompactWarps;
    mask_compact_kernel<<<blocks, kCompactThreads, 0, s>>>(m, g, 0, nullptr, -1, nullptr);
    g_launches.fetch_add(1);
    rc = cuda_err(cudaGetLastError());
    if (rc != LITE_OK) return rc;
    static_assert(sizeof(long long) == sizeof(int64_t), "live count width");
    return cuda_err(cudaMemcpyAsync(live_total, &scr->stats.live, sizeof(int64_t), cudaMemcpyDeviceToDevice, s));
}

#ifdef LITE_DEBUG_CHECKS
// Checked builds only: y_poly[i], y_mufu[i] = the two exponential paths of the
// attention kernel's softmax at x[i] (device arrays of n floats); synchronous.
int lite_attn_debug_exp2(const float *x, float *y_poly, float *y_mufu, int64_t n) {
    if (!x || !y_poly || !y_mufu || n < 1) return LITE_ERR_INVALID_ARG;
    const int blocks = static_cast<int>(std::min<int64_t>((n / 2 + 255) / 256 + 1, 148 * 8));
    exp2_paths_kernel<<<blocks, 256>>>(x, y_poly, y_mufu, n);
    g_launches.fetch_add(1);
    int rc = cuda_err(cudaGetLastError());
    if (rc == LITE_OK) rc = cuda_err(cudaDeviceSynchronize());
    return rc;
}
#endif

#ifdef LITE_PROFILE
// Profiling builds only: copy the per-CTA cycle counters to the host.
int lite_attn_debug_prof(void *host, size_t bytes) {
    if (bytes > sizeof(g_lite_prof)) bytes = sizeof(g_lite_prof);
    return cuda_err(cudaMemcpyFromSymbol(host, g_lite_prof, bytes));
}
int lite_attn_debug_trace(void *host, size_t bytes) {
    if (bytes > sizeof(g_lite_trace)) bytes = sizeof(g_lite_trace);
    return cuda_err(cudaMemcpyFromSymbol(host, g_lite_trace, bytes));
}
#endif

}  // extern "C"
