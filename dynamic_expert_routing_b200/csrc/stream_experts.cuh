// stream_experts.cuh -- weight-streaming SwiGLU experts for decode-sized groups (and the fp32
// layer), step 4 of the BEAM pipeline (BEAM article on aitrends.kr, masked aggregation), run
// only for the device-built list of groups with at least one kept slot, plus the always-on
// shared experts (same article, limitation (C)).
//
// For a handful of tokens per expert the expert FFN is a GEMV: every weight byte is used for
// at most a few FMAs, so the kernels are HBM-bound and are built to stream weights: 128-bit
// read-only loads, several independent loads in flight per lane, the group's activations
// staged in shared memory and reused for every weight row, split-K over the 32 lanes of a
// warp with a fixed butterfly reduction (deterministic, no atomics).
//
// Work items are (group, block of kStreamR weight rows); the shared group (when present)
// comes first.  A persistent grid walks the item list; groups with no kept token are absent
// from the list, so their weights are never read.
#pragma once
#include "common.cuh"

namespace beam {

constexpr int kStreamMT = 8;       // tokens per pass over a weight row
constexpr int kStreamR = 16;       // weight rows per work item
constexpr int kStreamWarps = 16;   // warps per CTA (one CTA per SM)
constexpr int kStreamThreads = 32 * kStreamWarps;
constexpr int kStreamNR = kStreamR / kStreamWarps;   // rows a warp streams at once
constexpr int kGuStreams = 2 * kStreamNR;            // gate/up: a gate and an up row per row
constexpr int kDnStreams = kStreamNR;                // down: one weight row per output row
static_assert(kStreamNR * kStreamWarps == kStreamR, "items split evenly over the warps");

struct StreamArgs {
    const void* xperm;   // routed activations, row g.row0 + i = i-th kept pair of group g
    const void* x;       // shared-expert activations [T][D]
    const void* wgu;     // routed gate/up [E][F/128][2][128][D] (gate block then up block)
    const void* wsgu;    // shared gate/up [Fsh/128][2][128][D]
    const void* wd;      // routed down [E][D][F], in the type of H
    const void* wsd;     // shared down [D][Fsh], in the type of H
    void* h;             // routed H [rows][F] (fp16 for bf16 layers, fp32 for fp32 layers)
    void* hsh;           // shared H [T][Fsh]
    float* yperm;        // routed Y [rows][D]
    float* ysh;          // shared Y [T][D]
    const Group* groups;
    const int* n_groups;
    int* err;            // error word of the forward's statistics
    int D, F, Fsh, T;
};

struct ItemView {
    const void* act;   // first activation row of the group
    int expert;        // routed expert index, -1 for the shared group
    void* hrow;        // first H row of the group
    float* yrow;       // first Y row of the group
    int m;             // rows (tokens) in the group
    int FF;            // intermediate size of the group
    int rb;            // row block inside the group
};

template <typename T, typename TH>
__device__ __forceinline__ ItemView stream_item(const StreamArgs& a, long item, int rb_shared,
                                                int rb_routed, int ng)
{
    ItemView v;
    if (item < rb_shared) {
        v.act = a.x; v.m = a.T; v.FF = a.Fsh; v.rb = (int)item;
        v.expert = -1; v.hrow = a.hsh; v.yrow = a.ysh;
    } else {
        const long r = item - rb_shared;
        const Group g = a.groups[r / rb_routed];
        v.rb = (int)(r % rb_routed);
        v.m = g.m; v.FF = a.F;
        v.act = static_cast<const T*>(a.xperm) + (size_t)g.row0 * a.D;
        v.hrow = static_cast<TH*>(a.h) + (size_t)g.row0 * a.F;
        v.yrow = a.yperm + (size_t)g.row0 * a.D;
        v.expert = g.expert;
    }
    return v;
}

// ---------------------------------------------------------------- warp-private TMA ring
// Each warp streams its weight rows through its own ring of kRingNS shared-memory stages,
// filled by 1-D bulk copies (cp.async.bulk, one per segment) that lane 0 issues kRingNS segments
// ahead of the computation; an mbarrier per stage signals arrival (transaction bytes).  A
// stage is refilled once every lane of the warp has read it (__syncwarp + proxy fence).
// This keeps kRingNS x (segment bytes) x (rows) in flight per warp independently of
// register pressure.  Segment k of a warp's stream always lands in stage k % kRingNS and its
// wait parity is (k / kRingNS) & 1.  Every wait is bounded in time.
constexpr int kRingNS = 4;
constexpr unsigned long long kRingWaitNs = 2000000000ull;
constexpr int ERR_STREAM_TIMEOUT = 0x200;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void ring_bar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar));
}
__device__ __forceinline__ void ring_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void ring_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ bool ring_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait; false (and the CTA-wide abort flag raised) on expiry or on an abort elsewhere.
__device__ __forceinline__ bool ring_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (ring_try(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!ring_try(bar, parity)) {
        if (*abort_flag) return false;
        if (gtimer() - t0 > kRingWaitNs) { *abort_flag = 1; return false; }
    }
    return true;
}
__device__ __forceinline__ void ring_release() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Issue segment c (elements [c*SEG, c*SEG + len)) of NQ rows into stage k % kRingNS.
template <typename T, int NQ>
__device__ __forceinline__ void ring_issue(uint32_t ring, uint32_t bars, int stage_bytes,
                                           int seg_bytes, long long k, const T* const* rows,
                                           int c, int SEG, int len)
{
    const int s = (int)(k % kRingNS);
    const uint32_t bar = bars + 8u * s;
    const uint32_t bytes = (uint32_t)(len * (int)sizeof(T));
    ring_expect(bar, bytes * NQ);
#pragma unroll
    for (int q = 0; q < NQ; ++q)
        ring_copy(ring + (uint32_t)(s * stage_bytes + q * seg_bytes), rows[q] + (size_t)c * SEG, bytes, bar);
}

// After an abort: let every copy a warp issued land before the CTA can exit.
__device__ __forceinline__ void ring_drain(uint32_t bars, long long issued, long long consumed) {
    for (long long k = consumed; k < issued; ++k) {
        const uint32_t bar = bars + 8u * (uint32_t)(k % kRingNS);
        const unsigned long long t0 = gtimer();
        while (!ring_try(bar, (uint32_t)((k / kRingNS) & 1)) && gtimer() - t0 < kRingWaitNs) {}
    }
}

constexpr int kGuSegBytes = 1024;    // bytes per row segment, gate/up kernel (kGuStreams per stage)
constexpr int kDnSegBytes = 2048;    // bytes per row segment, down kernel (kDnStreams per stage)
constexpr int kXTileBytes = 65536;   // activation tile of the gate/up kernel
constexpr int kHTileBytes = 81920;   // H tile of the down kernel

__host__ __device__ constexpr int stream_gateup_smem() {
    return kXTileBytes + kStreamWarps * kRingNS * kGuStreams * kGuSegBytes + kStreamWarps * kRingNS * 8 + 16;
}
__host__ __device__ constexpr int stream_down_smem() {
    return kHTileBytes + kStreamWarps * kRingNS * kDnStreams * kDnSegBytes + kStreamWarps * kRingNS * 8 + 16;
}

// Producer cursor of the gate/up kernel: position (item, pass p0, segment c) in the warp's
// segment stream, with the warp's kGuStreams weight rows of the item.  The consumer walks the same sequence,
// so the producer can run kRingNS segments ahead across item and pass boundaries.
template <typename T>
struct GuCursor {
    long item;
    int p0, c, m;
    const T* rows[kGuStreams];
    bool valid;
};

template <typename T, typename TH>
__device__ __forceinline__ void gu_rows(const StreamArgs& a, const ItemView& v, int warp,
                                        const T** rows)
{
    const T* wbase = v.expert < 0 ? static_cast<const T*>(a.wsgu)
                                  : static_cast<const T*>(a.wgu) + (size_t)v.expert * 2 * a.F * a.D;
    const int f0 = v.rb * kStreamR + warp * kStreamNR;
#pragma unroll
    for (int q = 0; q < kStreamNR; ++q) {
        const int f = f0 + q;
        rows[2 * q] = wbase + ((size_t)(f >> 7) * 256 + (f & 127)) * a.D;
        rows[2 * q + 1] = rows[2 * q] + (size_t)128 * a.D;
    }
}

// H[i][f] = silu(sum_d Wg[f][d] x_i[d]) * (sum_d Wu[f][d] x_i[d]) for the group's tokens i.
// T: storage type of x and the gate/up weights; TH: type of H.  Each warp owns kStreamNR
// intermediate rows of an item (kGuStreams weight streams: gate f, up f, ...).
template <typename T, typename TH>
__global__ void __launch_bounds__(kStreamThreads, 1)
stream_gateup_kernel(StreamArgs a)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int VN = Vec<T>::N;
    constexpr int SEG = kGuSegBytes / (int)sizeof(T);
    constexpr int STAGE = kGuStreams * kGuSegBytes;
    T* xs = reinterpret_cast<T*>(smem_raw);
    unsigned char* ring_p = smem_raw + kXTileBytes;
    uint64_t* bars_p = reinterpret_cast<uint64_t*>(ring_p + kStreamWarps * kRingNS * STAGE);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars_p + kStreamWarps * kRingNS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = smem_addr(ring_p) + (uint32_t)(warp * kRingNS * STAGE);
    const uint32_t bars = smem_addr(bars_p) + (uint32_t)(warp * kRingNS * 8);
    const unsigned char* ring_g = ring_p + warp * kRingNS * STAGE;
    if (lane == 0)
        for (int s = 0; s < kRingNS; ++s) ring_bar_init(bars + 8u * s);
    if (threadIdx.x == 0) *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    pdl_wait();

    const int D = a.D;
    const int MTX = min(kStreamMT, kXTileBytes / (D * (int)sizeof(T)));
    const int ng = *a.n_groups;
    const int rb_routed = a.F / kStreamR;
    const int rb_shared = a.Fsh / kStreamR;
    const long total = (long)rb_shared + (long)ng * rb_routed;
    const int nseg = (D + SEG - 1) / SEG;
    const void* cached = nullptr;
    int cached_rows = 0;
    // ok turns false (warp-uniformly) when a wait gives up; the warp then keeps walking the
    // same loops, so every __syncthreads is still reached, but issues and computes nothing.
    bool ok = true;

    // ---- producer (lane 0 issues; every lane keeps the cursor so the state stays uniform)
    GuCursor<T> pc;
    pc.item = blockIdx.x; pc.p0 = 0; pc.c = 0; pc.m = 0; pc.valid = false;
    auto load = [&]() {
        pc.valid = pc.item < total;
        if (pc.valid) {
            const ItemView v = stream_item<T, TH>(a, pc.item, rb_shared, rb_routed, ng);
            pc.m = v.m;
            gu_rows<T, TH>(a, v, warp, pc.rows);
        }
    };
    load();
    long long k_issue = 0, k_cons = 0;
    auto produce = [&]() {
        if (!ok || !pc.valid) return;
        if (lane == 0) {
            ring_release();
            ring_issue<T, kGuStreams>(ring, bars, STAGE, kGuSegBytes, k_issue, pc.rows, pc.c, SEG,
                                      min(SEG, D - pc.c * SEG));
        }
        ++k_issue;
        if (++pc.c == nseg) {
            pc.c = 0;
            pc.p0 += MTX;
            if (pc.p0 >= pc.m) { pc.p0 = 0; pc.item += gridDim.x; load(); }
        }
    };
    for (int i = 0; i < kRingNS; ++i) produce();

    // ---- consumer
    for (long item = blockIdx.x; item < total; item += gridDim.x) {
        const ItemView v = stream_item<T, TH>(a, item, rb_shared, rb_routed, ng);
        const int f0 = v.rb * kStreamR + warp * kStreamNR;
        for (int p0 = 0; p0 < v.m; p0 += MTX) {
            const int mp = min(MTX, v.m - p0);
            const T* src = static_cast<const T*>(v.act) + (size_t)p0 * D;
            if (src != cached || mp != cached_rows) {
                __syncthreads();
                const int nv = mp * D / VN;
                const uint4* s4 = reinterpret_cast<const uint4*>(src);
                uint4* d4 = reinterpret_cast<uint4*>(xs);
                for (int q = threadIdx.x; q < nv; q += blockDim.x) d4[q] = s4[q];
                __syncthreads();
                cached = src;
                cached_rows = mp;
            }
            float acc[kGuStreams][kStreamMT];
#pragma unroll
            for (int q = 0; q < kGuStreams; ++q)
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) acc[q][i] = 0.f;
            for (int c = 0; c < nseg && ok; ++c) {
                const long long k = k_cons;
                ok = __all_sync(0xffffffffu, ring_wait(bars + 8u * (uint32_t)(k % kRingNS),
                                                       (uint32_t)((k / kRingNS) & 1), abort_flag));
                if (!ok) break;
                const unsigned char* st = ring_g + (k % kRingNS) * STAGE;
                const int len = min(SEG, D - c * SEG);
                for (int e = lane * VN; e < len; e += 32 * VN) {
                    float w[kGuStreams][VN];
#pragma unroll
                    for (int q = 0; q < kGuStreams; ++q)
                        Vec<T>::widen(*reinterpret_cast<const uint4*>(st + q * kGuSegBytes + e * sizeof(T)), w[q]);
#pragma unroll
                    for (int i = 0; i < kStreamMT; ++i) {
                        if (i < mp) {
                            float xv[VN];
                            Vec<T>::widen(*reinterpret_cast<const uint4*>(xs + (size_t)i * D + c * SEG + e), xv);
#pragma unroll
                            for (int q = 0; q < kGuStreams; ++q) {
                                float sacc = 0.f;
#pragma unroll
                                for (int j = 0; j < VN; ++j) sacc = fmaf(w[q][j], xv[j], sacc);
                                acc[q][i] += sacc;
                            }
                        }
                    }
                }
                ++k_cons;
                __syncwarp();
                produce();
            }
            if (!ok) continue;
            TH* hout = static_cast<TH*>(v.hrow);
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q) {
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) {
                    if (i < mp) {
                        const float g = warp_sum(acc[2 * q][i]);
                        const float u = warp_sum(acc[2 * q + 1][i]);
                        if (lane == 0) {
                            const float hv = silu_f(g) * u;
                            if (sizeof(TH) == 2 && fp16_out_of_range(hv)) atomicOr(a.err, ERR_FP16_RANGE);
                            hout[(size_t)(p0 + i) * v.FF + f0 + q] = from_float<TH>(hv);
                        }
                    }
                }
            }
        }
    }
    if (!ok && lane == 0) {
        ring_drain(bars, k_issue, k_cons);
        atomicOr(a.err, ERR_STREAM_TIMEOUT);
    }
    pdl_launch_dependents();
}

// Largest H chunk (a whole number of segments) that fits the H tile for mp token rows.
template <typename T>
__device__ __forceinline__ int down_chunk(int mp, int SEG) {
    return max(SEG, (kHTileBytes / (mp * (int)sizeof(T))) / SEG * SEG);
}

// Y[i][j] = sum_f Wd[j][f] H[i][f] for the group's tokens i.  Each warp owns kDnStreams
// output rows of an item (one weight stream each).  H is staged in shared memory in chunks of up to
// kHTileBytes; the producer cursor runs across chunk, pass and item boundaries, so the next
// weight segments are already in flight while a chunk of H is being staged.
// T: type of H and of the down weights.
template <typename T>
__global__ void __launch_bounds__(kStreamThreads, 1)
stream_down_kernel(StreamArgs a)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    constexpr int VN = Vec<T>::N;
    constexpr int SEG = kDnSegBytes / (int)sizeof(T);
    constexpr int STAGE = kDnStreams * kDnSegBytes;
    T* hs = reinterpret_cast<T*>(smem_raw);
    unsigned char* ring_p = smem_raw + kHTileBytes;
    uint64_t* bars_p = reinterpret_cast<uint64_t*>(ring_p + kStreamWarps * kRingNS * STAGE);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars_p + kStreamWarps * kRingNS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ring = smem_addr(ring_p) + (uint32_t)(warp * kRingNS * STAGE);
    const uint32_t bars = smem_addr(bars_p) + (uint32_t)(warp * kRingNS * 8);
    const unsigned char* ring_g = ring_p + warp * kRingNS * STAGE;
    if (lane == 0)
        for (int s = 0; s < kRingNS; ++s) ring_bar_init(bars + 8u * s);
    if (threadIdx.x == 0) *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncthreads();
    pdl_wait();

    const int D = a.D;
    const int ng = *a.n_groups;
    const int rb_routed = D / kStreamR;
    const int rb_shared = a.Fsh > 0 ? D / kStreamR : 0;
    const long total = (long)rb_shared + (long)ng * rb_routed;
    bool ok = true;  // as in the gate/up kernel: a warp that gave up still reaches every barrier

    // ---- producer cursor: (item, pass p0, chunk start c0, segment c)
    struct {
        long item;
        int p0, c0, c, m, FF, cap;
        const T* rows[kDnStreams];
        bool valid;
    } pc;
    pc.item = blockIdx.x; pc.p0 = 0; pc.c0 = 0; pc.c = 0; pc.m = 0; pc.FF = 0; pc.cap = SEG;
    pc.valid = false;
    auto load = [&]() {
        pc.valid = pc.item < total;
        if (pc.valid) {
            const ItemView v = stream_item<T, T>(a, pc.item, rb_shared, rb_routed, ng);
            const T* wbase = v.expert < 0 ? static_cast<const T*>(a.wsd)
                                          : static_cast<const T*>(a.wd) + (size_t)v.expert * D * a.F;
            const int j0 = v.rb * kStreamR + warp * kStreamNR;
            pc.m = v.m;
            pc.FF = v.FF;
#pragma unroll
            for (int q = 0; q < kDnStreams; ++q) pc.rows[q] = wbase + (size_t)(j0 + q) * v.FF;
            pc.p0 = 0; pc.c0 = 0; pc.c = 0;
            pc.cap = down_chunk<T>(min(kStreamMT, pc.m), SEG);
        }
    };
    load();
    long long k_issue = 0, k_cons = 0;
    auto produce = [&]() {
        if (!ok || !pc.valid) return;
        const int fl = min(pc.cap, pc.FF - pc.c0);
        const int nseg = (fl + SEG - 1) / SEG;
        if (lane == 0) {
            const T* crow[kDnStreams];
#pragma unroll
            for (int q = 0; q < kDnStreams; ++q) crow[q] = pc.rows[q] + pc.c0;
            ring_release();
            ring_issue<T, kDnStreams>(ring, bars, STAGE, kDnSegBytes, k_issue, crow, pc.c, SEG,
                                      min(SEG, fl - pc.c * SEG));
        }
        ++k_issue;
        if (++pc.c == nseg) {
            pc.c = 0;
            pc.c0 += pc.cap;
            if (pc.c0 >= pc.FF) {
                pc.c0 = 0;
                pc.p0 += kStreamMT;
                if (pc.p0 >= pc.m) { pc.item += gridDim.x; load(); }
                else pc.cap = down_chunk<T>(min(kStreamMT, pc.m - pc.p0), SEG);
            }
        }
    };
    for (int i = 0; i < kRingNS; ++i) produce();

    // ---- consumer
    for (long item = blockIdx.x; item < total; item += gridDim.x) {
        const ItemView v = stream_item<T, T>(a, item, rb_shared, rb_routed, ng);
        const int FF = v.FF;
        const int j0 = v.rb * kStreamR + warp * kStreamNR;
        for (int p0 = 0; p0 < v.m; p0 += kStreamMT) {
            const int mp = min(kStreamMT, v.m - p0);
            const int cap = down_chunk<T>(mp, SEG);
            const T* hsrc = static_cast<const T*>(v.hrow) + (size_t)p0 * FF;
            float acc[kDnStreams][kStreamMT];
#pragma unroll
            for (int q = 0; q < kDnStreams; ++q)
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) acc[q][i] = 0.f;
            for (int c0 = 0; c0 < FF; c0 += cap) {
                const int fl = min(cap, FF - c0);
                const int nseg = (fl + SEG - 1) / SEG;
                __syncthreads();
                const int vpr = fl / VN;
                for (int q = threadIdx.x; q < mp * vpr; q += blockDim.x) {
                    const int i = q / vpr, cc = q - i * vpr;
                    reinterpret_cast<uint4*>(hs + (size_t)i * cap)[cc] =
                        reinterpret_cast<const uint4*>(hsrc + (size_t)i * FF + c0)[cc];
                }
                __syncthreads();
                for (int c = 0; c < nseg && ok; ++c) {
                    const long long k = k_cons;
                    ok = __all_sync(0xffffffffu, ring_wait(bars + 8u * (uint32_t)(k % kRingNS),
                                                           (uint32_t)((k / kRingNS) & 1), abort_flag));
                    if (!ok) break;
                    const unsigned char* st = ring_g + (k % kRingNS) * STAGE;
                    const int len = min(SEG, fl - c * SEG);
                    for (int e = lane * VN; e < len; e += 32 * VN) {
                        float w[kDnStreams][VN];
#pragma unroll
                        for (int q = 0; q < kDnStreams; ++q)
                            Vec<T>::widen(*reinterpret_cast<const uint4*>(st + q * kDnSegBytes + e * sizeof(T)), w[q]);
#pragma unroll
                        for (int i = 0; i < kStreamMT; ++i) {
                            if (i < mp) {
                                float hv[VN];
                                Vec<T>::widen(*reinterpret_cast<const uint4*>(hs + (size_t)i * cap + c * SEG + e), hv);
#pragma unroll
                                for (int q = 0; q < kDnStreams; ++q) {
                                    float sacc = 0.f;
#pragma unroll
                                    for (int j = 0; j < VN; ++j) sacc = fmaf(w[q][j], hv[j], sacc);
                                    acc[q][i] += sacc;
                                }
                            }
                        }
                    }
                    ++k_cons;
                    __syncwarp();
                    produce();
                }
            }
            if (!ok) continue;
#pragma unroll
            for (int q = 0; q < kDnStreams; ++q) {
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) {
                    if (i < mp) {
                        const float sum = warp_sum(acc[q][i]);
                        if (lane == 0) v.yrow[(size_t)(p0 + i) * D + j0 + q] = sum;
                    }
                }
            }
        }
    }
    if (!ok && lane == 0) {
        ring_drain(bars, k_issue, k_cons);
        atomicOr(a.err, ERR_STREAM_TIMEOUT);
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- combine
// y[t] = sum over slots k in rank order with keep = 1 of g_hat[t][k] * Y_perm[inv[t][k]],
// plus the shared-expert output; a fixed order, so the result is bit-reproducible.  When the
// down projection ran split-K, Y_perm / Y_sh hold `splits` partial slices `stride` elements
// apart (fp32), added in slice order before the gate is applied.  TY / TS are the element
// types of Y_perm / Y_sh: fp16 for unsplit tensor-core outputs of bf16 layers, fp32 otherwise.
__device__ __forceinline__ float4 load4(const float* p, size_t i) {
    return reinterpret_cast<const float4*>(p)[i];
}
__device__ __forceinline__ float4 load4(const __half* p, size_t i) {
    const uint2 u = reinterpret_cast<const uint2*>(p)[i];
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// y stores of 4 columns (streaming): float32, or rounded to bf16 (nearest even) for a
// BEAM_Y_BF16 forward.
__device__ __forceinline__ void store_y4(float* y, size_t i, float4 v)
{
    __stcs(reinterpret_cast<float4*>(y) + i, v);
}
__device__ __forceinline__ void store_y4(__nv_bfloat16* y, size_t i, float4 v)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a);
    o.y = *reinterpret_cast<const uint32_t*>(&b);
    __stcs(reinterpret_cast<uint2*>(y) + i, o);
}

template <typename TY, typename TS, typename TO = float>
__global__ void __launch_bounds__(256)
combine_kernel(const TY* __restrict__ yperm, int splits, long long stride,
               const TS* __restrict__ ysh, int splits_sh, long long stride_sh,
               const int* __restrict__ inv, const float* __restrict__ ghat, int T, int K, int D,
               TO* __restrict__ y)
{
    __shared__ int s_inv[32];
    __shared__ float s_g[32];
    pdl_wait();
    const int t = blockIdx.x;   // token; blockIdx.y picks a slice of the columns
    if (t >= T) return;
    if (threadIdx.x < K) {
        s_inv[threadIdx.x] = inv[(size_t)t * K + threadIdx.x];
        s_g[threadIdx.x] = ghat[(size_t)t * K + threadIdx.x];
    }
    __syncthreads();
    const int D4 = D >> 2;
    const long long s4 = stride >> 2, ssh4 = stride_sh >> 2;
    const int chunk = (D4 + gridDim.y - 1) / gridDim.y;   // columns of this CTA: one slice
    const int c_end = min(D4, (int)(blockIdx.y + 1) * chunk);
    for (int c = blockIdx.y * chunk + threadIdx.x; c < c_end; c += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // independent loads of up to 4 slots in flight before they are accumulated in order
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
            const int p = s_inv[k];
            if (p >= 0) {
                float4 v = load4(yperm, (size_t)p * D4 + c);
                for (int s = 1; s < splits; ++s) {
                    const float4 w = load4(yperm, s * s4 + (size_t)p * D4 + c);
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                const float g = s_g[k];
                acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
            }
        }
        if (ysh) {
            for (int s = 0; s < splits_sh; ++s) {
                const float4 w = load4(ysh, s * ssh4 + (size_t)t * D4 + c);
                acc.x += w.x; acc.y += w.y; acc.z += w.z; acc.w += w.w;
            }
        }
        store_y4(y, (size_t)t * D4 + c, acc);
    }
    pdl_launch_dependents();
}

// The combine of a small batch (fewer tokens than SMs) whose expert outputs are split-K slices:
// the per-column chain of slot x slice loads of combine_kernel is a long dependent walk there.
// CTA (token t, 16-column block) has 16 x (K + 1) threads: thread (c, k < K) adds the slices of
// slot k's row in slice order (their loads all issued first), thread (c, K) the slices of the
// shared term; then thread (c, 0) takes y = sum over the slots in rank order of g_hat * v_k
// (fmaf, as combine_kernel) + the shared sum.  Deterministic.  K <= 32, splits <= 16.
constexpr int kCombineSmallCols = 16;
constexpr int kCombineMaxSplits = 16;

template <typename TY>
__device__ __forceinline__ float4 sum_slices(const TY* base, int splits, long long s4, size_t i)
{
    float4 v[kCombineMaxSplits];
#pragma unroll
    for (int s = 0; s < kCombineMaxSplits; ++s)
        if (s < splits) v[s] = load4(base, s * s4 + i);
    float4 a = v[0];
#pragma unroll
    for (int s = 1; s < kCombineMaxSplits; ++s) {
        if (s < splits) { a.x += v[s].x; a.y += v[s].y; a.z += v[s].z; a.w += v[s].w; }
    }
    return a;
}

template <typename TY, typename TS, typename TO = float>
__global__ void __launch_bounds__(kCombineSmallCols * 33)
combine_small_kernel(const TY* __restrict__ yperm, int splits, long long stride,
                     const TS* __restrict__ ysh, int splits_sh, long long stride_sh,
                     const int* __restrict__ inv, const float* __restrict__ ghat, int T, int K,
                     int D, TO* __restrict__ y)
{
    __shared__ float4 red[33][kCombineSmallCols];
    __shared__ int s_inv[32];
    __shared__ float s_g[32];
    pdl_wait();
    const int t = blockIdx.x;
    const int cx = threadIdx.x, k = threadIdx.y;
    const int D4 = D >> 2;
    const int c = blockIdx.y * kCombineSmallCols + cx;
    const int tid = k * kCombineSmallCols + cx;
    if (tid < K) {
        s_inv[tid] = inv[(size_t)t * K + tid];
        s_g[tid] = ghat[(size_t)t * K + tid];
    }
    __syncthreads();
    if (c < D4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k < K) {
            const int p = s_inv[k];
            if (p >= 0) v = sum_slices(yperm, splits, stride >> 2, (size_t)p * D4 + c);
        } else if (ysh) {
            v = sum_slices(ysh, splits_sh, stride_sh >> 2, (size_t)t * D4 + c);
        }
        red[k][cx] = v;
    }
    __syncthreads();
    if (k == 0 && c < D4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 0; q < K; ++q) {
            if (s_inv[q] >= 0) {
                const float g = s_g[q];
                const float4 v = red[q][cx];
                acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
            }
        }
        if (ysh) {
            const float4 v = red[K][cx];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        store_y4(y, (size_t)t * D4 + c, acc);
    }
    pdl_launch_dependents();
}

}  // namespace beam
