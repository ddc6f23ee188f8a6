// tc_experts.cuh -- grouped SwiGLU experts on the 5th-generation tensor cores (tcgen05) for
// prefill-sized groups: step 4 of the BEAM pipeline (BEAM article on aitrends.kr, masked
// aggregation) over the device-built list of kept groups, plus the always-on shared experts
// (limitation (C)).  The expert FFN is a dense contraction, so it runs as two grouped GEMMs:
//   GEMM1  acc[t][0:128 | 128:256] = X_g[t] . [W_g rows | W_u rows]^T  ->  H = silu(gate) * up
//   GEMM2  Y_g[t][n] = H_g[t] . W_d[n]^T
// Design (sm_100a):
//   * one persistent CTA per SM walks a tile list derived on the device from the group table:
//     tiles are (problem, group, n tile, K split, m tile) with the m tile fastest, so CTAs
//     running at the same time share a weight tile through L2; groups with no kept token have
//     no tile, so their weights are never read;
//   * small batches split K across tiles so that a handful of kept groups still spreads over
//     every SM: the f32-store epilogue then writes per-split partial sums, which the next step
//     adds in a fixed order (the SwiGLU finishing kernel for gate/up, the combine for down);
//   * a group of at most 64 rows runs swapped (weights as the M = 128 operand, the group's rows
//     as N = 32 or 64, loaded as 32-row boxes): such a tile streams its weights alone, and the
//     swap cuts the activation copies from 16 to 4-8 KB per k-step.  (The short last tile of a
//     larger group keeps the normal form: there the tensor pipe is the bound, and N <= 64
//     instructions take longer per row than the full-width tile.);
//   * larger batches keep whole-K tiles, except for the last, partial wave: its tiles may be cut
//     into K pieces run on otherwise idle SMs.  Each piece stores an f32 partial; the epilogue
//     warp that arrives last at a sub-block (an atomic counter decides who, never the order)
//     adds the pieces' partials in piece order and runs the normal epilogue on the sum;
//   * tile 128 (tokens) x 256 x 64; each CTA issues its own TMA loads (cp.async.bulk.tensor,
//     128-byte swizzle) into a 4-stage shared-memory ring guarded by mbarriers;
//   * warp 0 lane 0 issues TMA, warp 1 lane 0 issues tcgen05.mma (kind::f16, fp32
//     accumulation in TMEM, double-buffered accumulators of 256 columns), warps 2..9 drain
//     TMEM with tcgen05.ld (two warps per lane quadrant, each half the columns) and run the
//     epilogue (SwiGLU -> fp16 H, or f32 / f16 stores);
//   * every mbarrier wait is bounded by a time limit; on expiry the CTA records an error code,
//     drains the copies and MMAs it issued (again bounded), frees TMEM and returns.
#pragma once
#include <cuda.h>
#include "common.cuh"

namespace beam {
namespace tc {

constexpr int BM = kGroupTileRows;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int kEpiWarps = 8;                 // two per TMEM lane quadrant, each half the columns
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer warp, MMA warp, epilogue warps
// Epilogue staging: each of the 4 epilogue warps transposes 32x32 fp32 sub-tiles through its
// own padded shared-memory buffer (row stride 33 words: conflict-free both ways).
constexpr int EPI_PITCH = 33;
constexpr int EPI_WARP_BYTES = 32 * EPI_PITCH * 4;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + kEpiWarps * EPI_WARP_BYTES + 1024 /*alignment slack*/ +
                           256 /*barriers*/;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s: far above any tile
// Swapped small groups: rows come in boxes of kSwapBox; groups of at most 2 boxes swap.
constexpr int kSwapBox = 32;
constexpr int SWAP_BOX_BYTES = kSwapBox * BK * 2;
// Tail split: at most kTailMaxPieces K pieces per tile, each at least kTailMinSteps k steps,
// spread over at most two sub-waves of the grid.  One piece's partial is one epilogue warp's
// 32 x 128 f32 sub-block per warp: kTailSlotFloats floats per (piece, warp).
constexpr int kTailMaxPieces = 8;
constexpr int kTailMinSteps = 8;
constexpr int kTailMaxSubWaves = 2;
constexpr int kTailSlotFloats = 4 * 32 * 32;
// Launches of fewer k steps use the kernel without the tail path: below 32 tail_pieces never
// splits (pieces of at least 8 steps that cut the tail by a quarter), and from 32 to 39 it
// splits only tails of at most a third of a wave, saving less than the heavier epilogue costs.
constexpr int kTailMinKSteps = 40;
constexpr int ERR_TC_TIMEOUT = 0x100;

// Epilogues: SwiGLU -> fp16 H; f32 stores (router logits, split-K partials); f16 stores
// (unsplit expert outputs Y_perm / Y_sh of bf16 layers).
enum Epi { EPI_SWIGLU = 0, EPI_STORE_F32 = 1, EPI_STORE_F16 = 2 };

struct TcParams {
    CUtensorMap a_routed;   // activations of the routed groups (rows = kept pairs)
    CUtensorMap b_routed;   // weights of the routed experts, [E * rows_per_expert][K]
    CUtensorMap a_shared;   // activations of the shared group (rows = tokens)
    CUtensorMap b_shared;   // shared-expert weights
    CUtensorMap a_routed_tail;  // a_routed with a kSwapBox-row box (swapped small groups)
    const Group* groups;
    const int* n_groups;    // [0]: groups, [1]: their tiles of BM rows
    const Group* tile_group;  // tile of BM rows (numbered across the groups) -> its group    // [0]: groups, [1]: their m tiles (tiles of BM rows)
    void* out_routed;       // EPI_SWIGLU: fp16 H [rows][F]; EPI_STORE_F32: f32 Y [rows][D]
    void* out_shared;
    int ld_routed;          // row length of out_routed
    int ld_shared;
    int b_rows_per_expert;  // 2F for GEMM1, D for GEMM2
    int n_tiles_routed;     // N / 256
    int n_tiles_shared;
    int k_steps_routed;     // K / 64
    int k_steps_shared;
    int k_splits_routed;    // split-K factor (1 = whole K per tile)
    int k_splits_shared;
    long long split_stride_routed;  // elements between the outputs of consecutive K splits
    long long split_stride_shared;
    int shared_rows;        // T, or 0 when there is no shared group
    int store_cols;         // f32 store epilogue: columns [0, store_cols) are stored (0 = all)
    int* err;
    // Tail split (whole-K launches of one problem only; null = off): arrival counters
    // [grid][kEpiWarps], zero on entry, and the partial workspace
    // [kTailMaxSubWaves * grid slots][kEpiWarps][kTailSlotFloats].
    int* tail_cnt;
    float* tail_ws;
    // SwiGLU folded into a split-K gate/up launch (EPI_STORE_F32 with the gate/up layout; null =
    // off): arrival counters [tiles][4 lane quadrants], zero between launches (the warp that
    // finishes a quadrant resets its counter), and the fp16 H outputs with their row lengths.
    int* fold_cnt;
    __half* fold_h_routed;
    __half* fold_h_shared;
    int fold_f_routed, fold_f_shared;
};

// Number of K pieces for the tail wave: rem whole-K tiles of ksteps k steps are left over after
// the full waves of a grid of G CTAs.  The estimated tail makespan, in k steps, is ksteps
// unsplit, and sub_waves * (ceil(ksteps / s) + 4 + 3 s) with s pieces (the constant covers the
// partial store and the fences, the 3 s the reading of s partials by the warp that finishes
// the sub-block).  A split must cut the estimate by at least a quarter; ties keep the smaller
// s.  Every thread of the grid evaluates this on the same integers.
__host__ __device__ inline int tail_pieces(long long rem, int ksteps, int G)
{
    if (rem <= 0) return 1;
    int best = 1;
    long long best_cost = ksteps;
    for (int s = 2; s <= kTailMaxPieces; ++s) {
        if (ksteps < kTailMinSteps * s) break;
        const long long sub = (rem * s + G - 1) / G;
        if (sub > kTailMaxSubWaves) break;
        const long long cost = sub * ((ksteps + s - 1) / s + 4 + 3 * s);
        if (cost < best_cost) { best_cost = cost; best = s; }
    }
    return 4 * best_cost <= 3LL * ksteps ? best : 1;
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait: false when the abort flag is raised elsewhere or the time limit passes (then
// this thread raises the flag itself).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            return false;
        }
    }
}

// Self-test of the bounded wait: one thread waits on an mbarrier whose phase nothing
// completes (its only expected arrival never comes), with a limit of limit_ns; the wait gives
// up, raises the abort flag, and the kernel records the outcome (2 = expired as designed,
// 0 = the phase completed, which cannot happen) and returns normally.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int* result)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
        *result = ok ? 0 : (abort_flag ? 2 : 1);
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 lanes x 32 consecutive fp32 columns of TMEM into 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), sm_100 version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;                 // leading byte offset (unused with swizzle): 16 B
    d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: 1024 B
    d |= (uint64_t)1 << 46;                 // descriptor version for sm_100
    d |= (uint64_t)2 << 61;                 // 128-byte swizzle
    return d;
}
// Instruction descriptor, kind::f16: fp32 accumulator, A/B of format `fmt` (0 = f16,
// 1 = bf16), both K-major, N = 256, M = 128.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t fmt, uint32_t n = BN) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((n >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

// ---------------------------------------------------------------- tile sequence
struct Tile {
    int shared;   // 1 = shared-expert problem
    int row0;     // first activation / output row of the group
    int m;        // rows in the group
    int mt;       // m tile inside the group
    int n;        // n tile
    int brow;     // first weight row of the tile
    int k0, k1;   // k steps [k0, k1) of this tile (its K split)
    int ks;       // K split index (selects the output slice)
    int gmt;      // m tile index across the launch's groups (routed), or inside the shared problem
    int swap;     // 0, or N (32 / 64): a swapped tail tile (weights = M operand, rows = N)
    int pieces;   // tail split: K pieces of this tile (1 = a whole tile)
    int tail;     // tail split: index of the tile among the split ones
    int slot;     // tail split: workspace slot of this piece (tail * pieces + piece)
};

__device__ __forceinline__ void split_range(int ksteps, int splits, int ks, int& k0, int& k1) {
    const int per = (ksteps + splits - 1) / splits;
    k0 = min(ksteps, ks * per);
    k1 = min(ksteps, k0 + per);
}

// Walks work units blockIdx.x, blockIdx.x + gridDim.x, ... in order; every role of a CTA
// holds its own copy and sees the same sequence.  Without a tail split a unit is a tile.  With
// one, units [0, whole_end) are the whole tiles of the full waves and the units after them the
// K pieces of the remaining tiles, tile-major (so tile indices never decrease along a walk).
// TAIL = false compiles the plain walk only; SWAP marks the groups of at most 64 rows.
template <bool TAIL, bool SWAP>
struct TileWalker {
    const TcParams* p;
    int total_mt;      // tiles of BM rows of the routed groups
    int count_sh;      // tiles of the shared problem
    int mts_sh;
    long long next;    // next unit index
    int whole_end;     // units below this are whole tiles
    int n_units;       // units of the launch
    int pieces;
    Group cg;          // the group of the last routed tile (most consecutive tiles share it)
    int cg_mts;

    // n_tiles: tiles of the launch (needed only with a tail split, else ignored)
    __device__ void init(const TcParams* p_, int total_mt_, long long n_tiles = 0) {
        p = p_;
        total_mt = total_mt_;
        mts_sh = p->shared_rows > 0 ? (p->shared_rows + BM - 1) / BM : 0;
        count_sh = mts_sh * p->n_tiles_shared * p->k_splits_shared;
        next = blockIdx.x;
        cg.mt0 = 0;
        cg_mts = 0;
        pieces = 1;
        whole_end = n_units = 0x7fffffff;
        if (TAIL && p->tail_cnt != nullptr) {
            const int ksteps = p->shared_rows > 0 ? p->k_steps_shared : p->k_steps_routed;
            const int rem = (int)(n_tiles % gridDim.x);
            pieces = tail_pieces(rem, ksteps, gridDim.x);
            if (pieces > 1) {
                whole_end = (int)(n_tiles - rem);
                n_units = whole_end + rem * pieces;
            }
        }
    }
    // tile index order inside a problem: m tile fastest, then K split, then n tile
    __device__ bool get(Tile& t) {
        const long long u = next;
        next += gridDim.x;
        long long i = u;
        int piece = 0;
        t.pieces = 1;
        t.tail = t.slot = 0;
        if (TAIL && u >= n_units) return false;
        if (TAIL && u >= whole_end) {
            const int local = (int)(u - whole_end);
            t.tail = local / pieces;
            piece = local % pieces;
            t.slot = local;
            t.pieces = pieces;
            i = whole_end + t.tail;
        }
        if (!locate(i, t)) return false;
        if (TAIL && t.pieces > 1) split_range(t.k1 - t.k0, t.pieces, piece, t.k0, t.k1);
        return true;
    }
    __device__ bool locate(long long i, Tile& t) {
        if (i < count_sh) {
            const int per_n = mts_sh * p->k_splits_shared;
            t.shared = 1;
            t.n = (int)(i / per_n);
            const int r = (int)(i % per_n);
            t.ks = r / mts_sh;
            t.mt = r % mts_sh;
            t.gmt = t.mt;
            t.row0 = 0;
            t.m = p->shared_rows;
            t.brow = t.n * BN;
            t.swap = 0;
            split_range(p->k_steps_shared, p->k_splits_shared, t.ks, t.k0, t.k1);
            return true;
        }
        // routed tiles: per group (n tile, K split, m tile), m fastest; a group's tiles start
        // at mt0 * tiles_per_mt, so tile i belongs to the group of m-tile i / tiles_per_mt
        const long long r = i - count_sh;
        const long long per_mt = (long long)p->n_tiles_routed * p->k_splits_routed;
        const long long q = r / per_mt;
        if (q >= total_mt) return false;
        if (q < cg.mt0 || q >= cg.mt0 + cg_mts) {
            cg = p->tile_group[q];
            cg_mts = (cg.m + BM - 1) / BM;
        }
        const long long rl = r - (long long)cg.mt0 * per_mt;
        const int per_n = cg_mts * p->k_splits_routed;
        t.shared = 0;
        t.n = (int)(rl / per_n);
        const int rr = (int)(rl % per_n);
        t.ks = rr / cg_mts;
        t.mt = rr % cg_mts;
        t.gmt = cg.mt0 + t.mt;
        t.row0 = cg.row0;
        t.m = cg.m;
        t.brow = cg.expert * p->b_rows_per_expert + t.n * BN;
        t.swap = (SWAP && cg.m <= 2 * kSwapBox) ? (cg.m <= kSwapBox ? kSwapBox : 2 * kSwapBox) : 0;
        split_range(p->k_steps_routed, p->k_splits_routed, t.ks, t.k0, t.k1);
        return true;
    }
};

// ---------------------------------------------------------------- the kernel
// Kernel forms.  MODE_TAIL: the launch may cut its last wave into K pieces (p.tail_cnt and
// p.tail_ws set).  MODE_SWAP: groups of at most 64 rows run swapped (p.a_routed_tail set).
// MODE_PLAIN has neither path compiled in.
enum Mode { MODE_PLAIN = 0, MODE_TAIL = 1, MODE_SWAP = 2 };

// Stores of one 32x32 f32 sub-tile from an epilogue warp's staging buffer (row i at
// buf + i * EPI_PITCH) to rows 0 .. nrows-1 of `out` (row pitch ld elements), 16 bytes per
// lane: fp16 takes 4 lanes per row, so one instruction writes 8 rows; f32 takes 8 lanes per
// row, 4 rows per instruction.  Lane l reads row-chunk (l / lanes_per_row, l % lanes_per_row):
// with the 33-word pitch the 32 lanes hit 32 different banks.  The column offset of `out`
// must be a multiple of 8 (fp16) or 4 (f32) elements and ld a multiple of the same.
__device__ __forceinline__ void store_rows_f16(const float* buf, __half* out, int ld, int nrows,
                                               int lane, bool& bad)
{
    const int cg = (lane & 3) * 8;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (8 * q >= nrows) break;   // warp-uniform: no rows left
        const int r = (lane >> 2) + 8 * q;
        if (r < nrows) {
            const float* s = buf + r * EPI_PITCH + cg;
            __half2 h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bad |= fp16_out_of_range(s[2 * j]) | fp16_out_of_range(s[2 * j + 1]);
                h[j] = __floats2half2_rn(s[2 * j], s[2 * j + 1]);
            }
            *reinterpret_cast<uint4*>(out + (size_t)r * ld + cg) = *reinterpret_cast<const uint4*>(h);
        }
    }
}

__device__ __forceinline__ void store_rows_f32(const float* buf, float* out, int ld, int nrows,
                                               int lane)
{
    const int cg = (lane & 7) * 4;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        if (4 * q >= nrows) break;   // warp-uniform: no rows left
        const int r = (lane >> 3) + 4 * q;
        if (r < nrows) {
            const float* s = buf + r * EPI_PITCH + cg;
            *reinterpret_cast<float4*>(out + (size_t)r * ld + cg) = make_float4(s[0], s[1], s[2], s[3]);
        }
    }
}

// Shared-memory layout of one CTA: [stage s: A (16 KB) | B (32 KB)] x STAGES, the epilogue
// staging buffers, then the mbarriers, the TMEM address slot and the abort flag.
struct GemmSmem {
    uint32_t base;              // shared-window address of the (1024-aligned) stage ring
    uint8_t* gbase;             // the same, generic
    float* epi_buf;
    uint32_t bar0;
    uint32_t* tmem_slot;
    volatile int* abort_flag;
    __device__ uint32_t full_bar(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t empty_bar(int s) const { return bar0 + 8u * (STAGES + s); }
    __device__ uint32_t tfull_bar(int a) const { return bar0 + 8u * (2 * STAGES + a); }
    __device__ uint32_t tempty_bar(int a) const { return bar0 + 8u * (2 * STAGES + 2 + a); }
    __device__ uint32_t drain_bar() const { return bar0 + 8u * (2 * STAGES + 4); }
};

__device__ __forceinline__ GemmSmem gemm_smem(uint8_t* smem_raw)
{
    GemmSmem m;
    const uint32_t raw = smem_u32(smem_raw);
    m.base = (raw + 1023u) & ~1023u;
    m.gbase = smem_raw + (m.base - raw);
    m.epi_buf = reinterpret_cast<float*>(m.gbase + STAGES * STAGE_BYTES);
    m.bar0 = m.base + STAGES * STAGE_BYTES + kEpiWarps * EPI_WARP_BYTES;
    m.tmem_slot = reinterpret_cast<uint32_t*>(m.gbase + STAGES * STAGE_BYTES + kEpiWarps * EPI_WARP_BYTES +
                                              8 * (2 * STAGES + 5));
    m.abort_flag = reinterpret_cast<volatile int*>(m.tmem_slot + 1);
    return m;
}

// Barrier init and TMEM allocation (warp 1), then a block barrier; returns the TMEM base.
__device__ __forceinline__ uint32_t gemm_setup(const GemmSmem& sm)
{
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(sm.full_bar(s), 1); mbar_init(sm.empty_bar(s), 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(sm.tfull_bar(a), 1); mbar_init(sm.tempty_bar(a), kEpiWarps); }
        mbar_init(sm.drain_bar(), 1);
        *sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(sm.tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return *sm.tmem_slot;
}

// After the last GEMM phase: a block barrier, the error word on an abort, TMEM freed.
__device__ __forceinline__ void gemm_teardown(const GemmSmem& sm, uint32_t tmem_base, int* err)
{
    const int warp = threadIdx.x >> 5;
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *sm.abort_flag) atomicOr(err, ERR_TC_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
    }
}

// Pipeline position of the thread playing a role (producer: stage s / phase ph; MMA issuer:
// stage, phase, accumulator acc / aph; epilogue: acc / aph).  It carries over from one GEMM
// phase of a launch to the next, as the mbarriers do.
struct RoleState {
    int s = 0, acc = 0;
    uint32_t ph = 0, aph = 0;
    bool ok = true, issued = false;
    int pend_ph[STAGES] = {0, 0, 0, 0};
    bool pend[STAGES] = {false, false, false, false};
};

// One GEMM phase over the tile list of `p`: warp 0 lane 0 issues TMA, warp 1 lane 0 issues
// MMAs, warps 2.. run the epilogue.  Returns with every tile of this CTA stored (or with
// rs.ok = false and the abort flag raised after a wait ran out, its copies and MMAs drained).
template <int EPI, int FMT, int MODE>
__device__ __forceinline__ void gemm_roles(const TcParams& p, const GemmSmem& sm,
                                           uint32_t tmem_base, RoleState& rs)
{
    constexpr bool TAIL = MODE == MODE_TAIL;
    constexpr bool SWAP = MODE == MODE_SWAP && EPI != EPI_STORE_F32;
    const uint32_t base = sm.base;
    float* epi_buf = sm.epi_buf;
    volatile int* abort_flag = sm.abort_flag;
    auto full_bar = [&](int s) { return sm.full_bar(s); };
    auto empty_bar = [&](int s) { return sm.empty_bar(s); };
    auto tfull_bar = [&](int a) { return sm.tfull_bar(a); };
    auto tempty_bar = [&](int a) { return sm.tempty_bar(a); };
    const uint32_t drain_bar = sm.drain_bar();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_mt = p.n_groups[1];
    // tiles of the launch (used by the tail split): n_groups[1] holds the groups' m tiles
    long long n_tiles = 0;
    if (TAIL && p.tail_cnt != nullptr) {
        const long long mts_sh = p.shared_rows > 0 ? (p.shared_rows + BM - 1) / BM : 0;
        n_tiles = (long long)total_mt * p.n_tiles_routed + mts_sh * p.n_tiles_shared;
    }

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        TileWalker<TAIL, SWAP> w;
        w.init(&p, total_mt, n_tiles);
        Tile t;
        int s = rs.s;
        uint32_t ph = rs.ph;
        bool ok = rs.ok;
        int* pend_ph = rs.pend_ph;
        bool* pend = rs.pend;
        while (ok && w.get(t)) {
            const CUtensorMap* am = t.shared ? &p.a_shared : &p.a_routed;
            const CUtensorMap* bm = t.shared ? &p.b_shared : &p.b_routed;
            const int arow = t.row0 + t.mt * BM;
            const int nbox = t.swap / kSwapBox;  // swapped tile: 1 or 2 boxes of rows
            for (int k = t.k0; k < t.k1; ++k) {
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag)) { ok = false; break; }
                const uint32_t sa = base + s * STAGE_BYTES;
                if (SWAP && t.swap) {
                    mbar_expect_tx(full_bar(s), B_BYTES + nbox * SWAP_BOX_BYTES);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(sa + b * SWAP_BOX_BYTES, &p.a_routed_tail, full_bar(s), k * BK,
                                    arow + b * kSwapBox);
                } else {
                    mbar_expect_tx(full_bar(s), STAGE_BYTES);
                    tma_load_2d(sa, am, full_bar(s), k * BK, arow);
                }
                tma_load_2d(sa + A_BYTES, bm, full_bar(s), k * BK, t.brow);
                pend[s] = true;
                pend_ph[s] = (int)ph;
                if (++s == STAGES) { s = 0; ph ^= 1u; }
            }
        }
        if (!ok && rs.ok) {
            // drain: let every copy this thread issued land before the CTA can exit
            for (int i = 0; i < STAGES; ++i) {
                if (!pend[i]) continue;
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(full_bar(i), (uint32_t)pend_ph[i]) &&
                       globaltimer() - t0 < kWaitLimitNs) {}
            }
        }
        rs.s = s; rs.ph = ph; rs.ok = ok;
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        TileWalker<TAIL, SWAP> w;
        w.init(&p, total_mt, n_tiles);
        Tile t;
        int s = rs.s, acc = rs.acc;
        uint32_t ph = rs.ph, aph = rs.aph;
        bool ok = rs.ok, issued = rs.issued;
        constexpr uint32_t idesc = make_idesc(FMT);
        while (ok && w.get(t)) {
            if (!mbar_wait(tempty_bar(acc), aph ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
            for (int k = t.k0; k < t.k1; ++k) {
                if (!mbar_wait(full_bar(s), ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = base + s * STAGE_BYTES;
                const uint64_t ad = sw128_desc(sa);
                const uint64_t bd = sw128_desc(sa + A_BYTES);
                if (SWAP && t.swap) {
                    // D[weight row][token]: each 128-row half of the weight tile is an M = 128
                    // operand; the tokens are the N operand; half h accumulates at column h*N
                    const uint32_t idesc_s = make_idesc(FMT, (uint32_t)t.swap);
                    const uint64_t wd1 = sw128_desc(sa + A_BYTES + BM * 128);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t accum = (k != t.k0 || kk != 0) ? 1u : 0u;
                        tc_mma_f16(d_tmem, bd + 2ull * kk, ad + 2ull * kk, idesc_s, accum);
                        tc_mma_f16(d_tmem + (uint32_t)t.swap, wd1 + 2ull * kk, ad + 2ull * kk, idesc_s, accum);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma_f16(d_tmem, ad + 2ull * kk, bd + 2ull * kk, idesc,
                                   (k != t.k0 || kk != 0) ? 1u : 0u);
                }
                issued = true;
                tc_commit(empty_bar(s));
                if (++s == STAGES) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
            tc_commit(tfull_bar(acc));
            if (++acc == 2) { acc = 0; aph ^= 1u; }
        }
        if (!ok && rs.ok && issued) {
            tc_commit(drain_bar);  // completes when every MMA issued so far has finished
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < kWaitLimitNs) {}
        }
        rs.s = s; rs.ph = ph; rs.acc = acc; rs.aph = aph; rs.ok = ok; rs.issued = issued;
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (TMEM -> registers -> global)
        TileWalker<TAIL, SWAP> w;
        w.init(&p, total_mt, n_tiles);
        Tile t;
        int acc = rs.acc;
        uint32_t aph = rs.aph;
        bool ok = rs.ok;
        bool bad = false;                // an fp16 store of this thread was out of range
        const int lb = 32 * (warp & 3);  // TMEM lanes this warp may access
        const int warp_e = warp - 2;     // index of this epilogue warp (its staging buffer)
        const int half = warp_e / 4;     // which half of the tile's columns this warp drains
        // TMEM column of chunk c (0..3) of this warp's sub-block: 32-column chunks of its half
        // of the tile; for SwiGLU the even chunks are gate columns, the odd ones the matching
        // up columns.
        auto chunk_col = [&](int c) {
            return EPI == EPI_SWIGLU ? (c & 1) * (BN / 2) + 32 * (half * 2 + (c >> 1))
                                     : 32 * (half * 4 + c);
        };
        while (ok && w.get(t)) {
            if (!mbar_wait(tfull_bar(acc), aph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)lb << 16) + (uint32_t)(acc * BN);
            // rows lb .. lb+31 of the tile belong to this warp; row_ok(i) = row i of them is
            // a row of the group.  Each 32-column chunk goes TMEM -> registers (thread = row)
            // -> padded shared memory -> registers (thread = column) -> one coalesced store per
            // row, so every store instruction writes one contiguous row segment.
            const int r0 = t.mt * BM + lb;                 // first row of this warp, in the group
            const int nrows = max(0, min(32, t.m - r0));   // valid rows of this warp
            float* buf = epi_buf + warp_e * (32 * EPI_PITCH);
            const int ld = t.shared ? p.ld_shared : p.ld_routed;
            const size_t row_base = (size_t)(t.row0 + r0);
            // Swapped tile (a small group): TMEM lane = weight row (feature), column = token.  Gate/up:
            // gate of the 128 features at columns [0, N), up at [N, 2N); warp half h takes the
            // tokens [32h, 32h + 32).  Down: features 128h + lane at columns [hN, hN + N).  Every
            // store writes 32 consecutive features of one token row.
            if (SWAP && t.swap) {
                const int N = t.swap;
                const int r_first = t.mt * BM;   // first row of the tile, in the group
                const uint32_t tb = tmem_base + ((uint32_t)lb << 16) + (uint32_t)(acc * BN);
                __half* out = static_cast<__half*>(t.shared ? p.out_shared : p.out_routed);
                if (EPI == EPI_SWIGLU) {
                    if (32 * half < N) {
                        float g[32], u[32];
                        tmem_ld32(tb + 32 * half, g);
                        tmem_ld32(tb + N + 32 * half, u);
                        const int r0h = r_first + 32 * half;
                        const int nr = max(0, min(32, t.m - r0h));
                        __half* col = out + (size_t)(t.row0 + r0h) * ld + (size_t)t.n * (BN / 2) + lb + lane;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i < nr) {
                                const float hv = silu_f(g[i]) * u[i];
                                bad |= fp16_out_of_range(hv);
                                *col = __float2half_rn(hv);
                            }
                            col += ld;
                        }
                    }
                } else {
#pragma unroll 1
                    for (int c = 0; c < N; c += 32) {
                        float v[32];
                        tmem_ld32(tb + half * N + c, v);
                        const int nr = max(0, min(32, t.m - r_first - c));
                        __half* col = out + (size_t)(t.row0 + r_first + c) * ld + (size_t)t.n * BN +
                                      half * BM + lb + lane;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i < nr) {
                                bad |= fp16_out_of_range(v[i]);
                                *col = __float2half_rn(v[i]);
                            }
                            col += ld;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(acc));
                if (++acc == 2) { acc = 0; aph ^= 1u; }
                continue;
            }
            // A K piece of a tail tile stores this warp's partial sub-block, frees the TMEM
            // buffer and counts the arrival; the warp that completes the count adds the
            // pieces' partials in piece order (red != null) and runs the epilogue on the sum.
            // Partial layout per (piece, warp): [chunk c][column i][row lane], so that a warp
            // writes and reads 32 consecutive floats per column.
            const float* red = nullptr;
            if (TAIL && t.pieces > 1) {
                float* mine = p.tail_ws + ((size_t)t.slot * kEpiWarps + warp_e) * kTailSlotFloats;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(tbase + chunk_col(c), v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) __stcg(mine + (c * 32 + i) * 32 + lane, v[i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(acc));
                if (++acc == 2) { acc = 0; aph ^= 1u; }
                __threadfence();
                __syncwarp();
                int prev = 0;
                if (lane == 0) prev = atomicAdd(p.tail_cnt + t.tail * kEpiWarps + warp_e, 1);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev != t.pieces - 1) continue;
                __syncwarp();
                __threadfence();   // the other pieces' partials are visible past this point
                red = p.tail_ws + ((size_t)t.tail * t.pieces * kEpiWarps + warp_e) * kTailSlotFloats;
            }
            // chunk c of this warp's rows (thread = row) summed over the pieces, in piece order
            auto reduce = [&](int c, float* v) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
                const float* src = red + c * 32 * 32 + lane;
#pragma unroll 1
                for (int q = 0; q < t.pieces; ++q, src += (size_t)kEpiWarps * kTailSlotFloats) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] += __ldcg(src + i * 32);
                }
            };
            if (EPI == EPI_SWIGLU) {
                __half* out = static_cast<__half*>(t.shared ? p.out_shared : p.out_routed);
#pragma unroll 1
                for (int j = half * (BN / 2 / 64); j < (half + 1) * (BN / 2 / 64); ++j) {
                    if (!TAIL || red == nullptr) {
                        float g[32], u[32];
                        tmem_ld32(tbase + 32 * j, g);
                        tmem_ld32(tbase + BN / 2 + 32 * j, u);
#pragma unroll
                        for (int i = 0; i < 32; ++i) buf[lane * EPI_PITCH + i] = silu_f(g[i]) * u[i];
                    } else {
                        // two passes keep 32 sums live: silu(gate) into the buffer, then * up
                        const int c = 2 * (j - half * (BN / 2 / 64));
                        float v[32];
                        reduce(c, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) buf[lane * EPI_PITCH + i] = silu_f(v[i]);
                        reduce(c + 1, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) buf[lane * EPI_PITCH + i] *= v[i];
                    }
                    __syncwarp();
                    store_rows_f16(buf, out + row_base * ld + (size_t)t.n * (BN / 2) + 32 * j, ld, nrows, lane, bad);
                    __syncwarp();
                }
            } else {
                const long long sstride = t.shared ? p.split_stride_shared : p.split_stride_routed;
#pragma unroll 1
                for (int j = half * (BN / 64); j < (half + 1) * (BN / 64); ++j) {
                    // the router's logit rows are padded to the tile width: only the chunks
                    // holding the 2E real columns are read back
                    if (EPI == EPI_STORE_F32 && p.store_cols > 0 && t.n * BN + 32 * j >= p.store_cols)
                        continue;
                    float v[32];
                    if (!TAIL || red == nullptr) tmem_ld32(tbase + 32 * j, v);
                    else reduce(j - half * (BN / 64), v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) buf[lane * EPI_PITCH + i] = v[i];
                    __syncwarp();
                    const size_t off = (size_t)t.ks * sstride + row_base * ld + (size_t)t.n * BN + 32 * j;
                    if (EPI == EPI_STORE_F16)
                        store_rows_f16(buf, static_cast<__half*>(t.shared ? p.out_shared : p.out_routed) + off,
                                       ld, nrows, lane, bad);
                    else
                        store_rows_f32(buf, static_cast<float*>(t.shared ? p.out_shared : p.out_routed) + off,
                                       ld, nrows, lane);
                    __syncwarp();
                }
            }
            if (!TAIL || red == nullptr) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(acc));
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
            if (EPI == EPI_STORE_F32 && p.fold_cnt != nullptr) {
                // SwiGLU folded into the split-K gate/up launch: the 2 warps of this lane
                // quadrant x the launch's K slices each store a partial; the warp whose arrival
                // completes the count (the atomic only elects it) adds the slices in slice order
                // and writes H = silu(gate) * up for the quadrant's rows and the tile's 128
                // features -- the same sums, in the same order, as the SwiGLU finishing kernel.
                const int splits = t.shared ? p.k_splits_shared : p.k_splits_routed;
                const long long mts_routed = p.n_groups[1];
                const long long tile = t.shared
                    ? mts_routed * p.n_tiles_routed + (long long)t.gmt * p.n_tiles_shared + t.n
                    : (long long)t.gmt * p.n_tiles_routed + t.n;
                int* cnt = p.fold_cnt + tile * 4 + (warp & 3);
                __threadfence();
                __syncwarp();
                int prev = 0;
                if (lane == 0) prev = atomicAdd(cnt, 1);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == 2 * splits - 1) {
                    __threadfence();   // the other partials of the quadrant are visible
                    const float* part = static_cast<const float*>(t.shared ? p.out_shared : p.out_routed);
                    const long long st = t.shared ? p.split_stride_shared : p.split_stride_routed;
                    __half* hout = t.shared ? p.fold_h_shared : p.fold_h_routed;
                    const int FF = t.shared ? p.fold_f_shared : p.fold_f_routed;
                    for (int i = 0; i < nrows; ++i) {
                        const size_t row = row_base + i;
                        const float* src = part + row * ld + (size_t)t.n * BN + 4 * lane;
                        float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
                        for (int q = 0; q < splits; ++q) {
                            const float4 a = __ldcg(reinterpret_cast<const float4*>(src + q * st));
                            const float4 b = __ldcg(reinterpret_cast<const float4*>(src + q * st + BN / 2));
                            g.x += a.x; g.y += a.y; g.z += a.z; g.w += a.w;
                            u.x += b.x; u.y += b.y; u.z += b.z; u.w += b.w;
                        }
                        const float h0 = silu_f(g.x) * u.x, h1 = silu_f(g.y) * u.y;
                        const float h2 = silu_f(g.z) * u.z, h3 = silu_f(g.w) * u.w;
                        bad |= fp16_out_of_range(h0) | fp16_out_of_range(h1) |
                               fp16_out_of_range(h2) | fp16_out_of_range(h3);
                        __half2 hv[2] = {__floats2half2_rn(h0, h1), __floats2half2_rn(h2, h3)};
                        *reinterpret_cast<uint2*>(hout + row * FF + (size_t)t.n * (BN / 2) + 4 * lane) =
                            *reinterpret_cast<const uint2*>(hv);
                    }
                    if (lane == 0) *cnt = 0;   // ready for the next launch
                }
            }
        }
        if (bad) atomicOr(p.err, ERR_FP16_RANGE);
        rs.acc = acc; rs.aph = aph; rs.ok = ok;
    }

}

template <int EPI, int FMT, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_gemm_kernel(const __grid_constant__ TcParams p)
{
    constexpr bool SWAP = MODE == MODE_SWAP && EPI != EPI_STORE_F32;
    extern __shared__ uint8_t smem_raw[];
    const GemmSmem sm = gemm_smem(smem_raw);
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&p.a_routed); tma_prefetch_desc(&p.b_routed);
        tma_prefetch_desc(&p.a_shared); tma_prefetch_desc(&p.b_shared);
        if (SWAP) tma_prefetch_desc(&p.a_routed_tail);
    }
    const uint32_t tmem_base = gemm_setup(sm);
    pdl_wait();  // groups, counts and activations come from the previous kernels
    RoleState rs;
    gemm_roles<EPI, FMT, MODE>(p, sm, tmem_base, rs);
    gemm_teardown(sm, tmem_base, p.err);
    pdl_launch_dependents();
}

}  // namespace tc
}  // namespace beam
