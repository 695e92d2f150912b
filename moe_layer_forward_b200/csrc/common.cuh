// Device helpers shared by the MoE layer kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

enum : int { DT_F32 = 0, DT_BF16 = 1 };
enum : int { DEV_BAD_EXPERT_ID = 1, DEV_TIMEOUT = 2, DEV_BAD_COUNT = 4 };

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }
__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// two floats -> packed bf16x2 (lo in the low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16);
}

// 8 consecutive elements of a row, as fp32 (x is f32 or bf16); p is 16-byte aligned
template <int DT>
__device__ __forceinline__ void load8(const void* base, int64_t elem, float (&o)[8]) {
    if constexpr (DT == DT_BF16) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem));
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
            o[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
        float4 a = __ldg(p), b = __ldg(p + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

template <int DT>
__device__ __forceinline__ void store8(void* base, int64_t elem, const float (&v)[8]) {
    if constexpr (DT == DT_BF16) {
        uint4 u;
        u.x = pack_bf16x2(v[0], v[1]);
        u.y = pack_bf16x2(v[2], v[3]);
        u.z = pack_bf16x2(v[4], v[5]);
        u.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(base) + elem) = u;
    } else {
        float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + elem);
        p[0] = make_float4(v[0], v[1], v[2], v[3]);
        p[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// raw 16-byte copies (8 bf16 or 4 f32)
__device__ __forceinline__ uint4 ld16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Programmatic dependent launch: wait for the preceding kernel's results /
// let the next kernel start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
    if (status) atomicOr(status, bits);
}

// Expert segment [off, off + cnt) as given, cut to the rows [0, S) of the buffer: (o, n) is the
// intersection.  Returns false when the given segment does not lie inside the buffer (negative count or
// offset, or past its end); the caller flags DEV_BAD_COUNT.
__device__ __forceinline__ bool clamp_segment(int off, int cnt, int S, int& o, int& n) {
    const bool ok = off >= 0 && cnt >= 0 && (int64_t)off + cnt <= (int64_t)S;
    const int64_t lo = off < 0 ? 0 : (off > S ? S : off);
    int64_t hi = cnt < 0 ? lo : (int64_t)off + cnt;
    if (hi > S) hi = S;
    o = (int)lo;
    n = hi > lo ? (int)(hi - lo) : 0;
    return ok;
}

}  // namespace moe
