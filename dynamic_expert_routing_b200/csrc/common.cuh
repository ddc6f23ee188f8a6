// common.cuh -- small device helpers shared by the BEAM kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace beam {

constexpr int kWarp = 32;

// One routed group = the kept (token, slot) pairs of one expert, contiguous in the permuted
// activation matrix: rows [row0, row0 + m) of X_perm / H / Y_perm belong to expert `expert`.
// Its tiles of kGroupTileRows rows are numbered mt0, mt0 + 1, ... across all groups in order.
struct __align__(16) Group {
    int row0;
    int m;
    int expert;
    int mt0;
};
static_assert(sizeof(Group) == 16, "Group is read as one 16-byte vector");

// Device-side statistics of one forward, reduced in a fixed order.
// Row-tile height of the tensor-core grouped GEMMs.  The compaction records, next to the
// number of groups, how many tiles of this height the groups take (the GEMMs' tile count).
constexpr int kGroupTileRows = 128;

struct DevStats {
    long long keep_sum;   // sum over tokens of kept slots
    double lreg_sum;      // sum over tokens of (1/K) sum_{TK} sigmoid(mask logit)
    int n_active;         // experts with >= 1 kept slot
    int n_all_masked;     // tokens with no kept slot
    int n_kept;           // kept (token, slot) pairs
    int tokens;
    int err;              // nonzero when a bounded wait ran out
    unsigned grid_bar;    // arrival counter, zeroed with err every forward: the fused decode
                          // kernel's grid barriers, or compact_scan's last-CTA election
};

// ---------------------------------------------------------------- storage-type helpers
// Exact widening of a pair of bf16 values packed in one 32-bit word (low half first).
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <typename T> struct Vec;  // 16-byte vector of storage elements
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void widen(const uint4& v, float* o) {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void widen(const uint4& v, float* o) {
        o[0] = bf16lo(v.x); o[1] = bf16hi(v.x); o[2] = bf16lo(v.y); o[3] = bf16hi(v.y);
        o[4] = bf16lo(v.z); o[5] = bf16hi(v.z); o[6] = bf16lo(v.w); o[7] = bf16hi(v.w);
    }
};

template <> struct Vec<__half> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void widen(const uint4& v, float* o) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            o[2 * i] = f.x;
            o[2 * i + 1] = f.y;
        }
    }
};

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_float(float v);
template <> __device__ __forceinline__ float from_float<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ __half from_float<__half>(float v) {
    return __float2half_rn(v);
}

// Type of the SwiGLU intermediate H for a storage type: fp32 layers keep fp32; bf16 layers
// use fp16, whose 10-bit mantissa rounds H eight times more finely than bf16 (the down
// projection then runs in fp16 x fp16 with fp32 accumulation).
template <typename TX> struct HType { using type = float; };
template <> struct HType<__nv_bfloat16> { using type = __half; };

// fp16 range of the stored intermediates (H = silu(gate) * up and the unsplit expert outputs
// of bf16 layers): a value that rounds to a finite fp16 has magnitude below 65520 (the midpoint
// between the largest fp16, 65504, and the next power of two).  A kernel that stores a value
// outside that range (or a NaN) sets this bit in the forward's error word; beam_moe_stats then
// reports BEAM_ERR_RANGE instead of returning numbers that hold an infinity.
constexpr int ERR_FP16_RANGE = 0x400;
__device__ __forceinline__ bool fp16_out_of_range(float v) { return !(fabsf(v) < 65520.0f); }

// Streaming 16-byte load through the read-only path, not kept in L1.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }

// Programmatic dependent launch: wait for the producer grid's memory to be visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace beam
