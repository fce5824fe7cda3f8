// Device helpers shared by the libcsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

constexpr int kRopeDims = 64;

__device__ __forceinline__ void flag(int32_t* st, int bits) {
    if (st) atomicOr(st, bits);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// Two packed bf16 (low half = first element) -> two floats.
__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t packed) {
    return make_float2(__uint_as_float(packed << 16), __uint_as_float(packed & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return (uint32_t)(*reinterpret_cast<uint16_t*>(&h));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return f32_to_bf16_bits(lo) | (f32_to_bf16_bits(hi) << 16);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    __nv_fp8_e4m3 v;
    v.__x = (__nv_fp8_storage_t)code;
    return float(v);
}

__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float x) {
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// RoPE rotation of pair j (of the last 64 dims) at position pos: cos/sin of
// pos * theta^(-2j/64).  The angle is formed and reduced to [-pi, pi] in fp64 so that
// positions up to 2^20 keep ~1e-7 rad accuracy; the reduced angle then goes to sincosf.
__device__ __forceinline__ void rope_cos_sin(double pos, int j, double log2_theta, float& c,
                                             float& s) {
    const double kTwoPi = 6.283185307179586476925;
    const double kInvTwoPi = 0.159154943091895335769;
    double inv_freq = exp2(-(double)(2 * j) * (1.0 / 64.0) * log2_theta);
    double a = pos * inv_freq;
    double r = a - kTwoPi * rint(a * kInvTwoPi);
    sincosf((float)r, &s, &c);
}

// Programmatic dependent launch.  Every libcsa kernel is launched so that it may start
// while the previous kernel on the stream finishes.  pdl_wait() blocks the calling thread
// until the previous grid has completed and its writes are visible; it must precede any
// read of data an earlier kernel produces and any write that an earlier kernel may still
// read.  pdl_trigger() lets the next kernel start launching; kernels issue it only after
// their own wait, so at most two kernels ever overlap.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Where the classical cache holds entry i of sequence b ("DeepSeek-V4 深度分析报告" 3.5: the
// compressed entries are managed in blocks of lcm(m, m') = 128 tokens).  Without a block
// table: row ent_off[b] + i of a contiguous per-sequence array.  With one: entry i lies in
// the sequence's block i / E (E = 128 / m entries per block, E = 2^pe_shift), at row
// bt[b * bt_stride + i / E] * E + i % E.
struct EntryRows {
    const int64_t* ent_off;
    const int32_t* bt;       // nullable
    int64_t bt_stride;
    int pe_shift;
    __device__ __forceinline__ int64_t row(int b, int64_t i) const {
        if (!bt) return ent_off[b] + i;
        const int64_t blk = bt[(int64_t)b * bt_stride + (i >> pe_shift)];
        return (blk << pe_shift) + (i & ((1ll << pe_shift) - 1));
    }
};

// Where the state cache holds raw token p of sequence b.  Linear (ring = 0): row
// kv_off[b] + p - kv_pos0[b], positions kv_pos0[b] .. seq_len[b] - 1 stored.  Ring
// (ring > 0): a fixed-size ring of `ring` rows per sequence, row kv_off[b] + p mod ring,
// positions max(seq_len[b] - ring, 0) .. seq_len[b] - 1 stored.
struct RawRows {
    const int64_t* kv_off;
    const int64_t* kv_pos0;  // unused with a ring
    int64_t ring;
    __device__ __forceinline__ int64_t first(int b, int64_t seq_len_b) const {
        if (ring) return seq_len_b > ring ? seq_len_b - ring : 0;
        return kv_pos0[b];
    }
    __device__ __forceinline__ int64_t row(int b, int64_t p) const {
        return ring ? kv_off[b] + p % ring : kv_off[b] + p - kv_pos0[b];
    }
};

// Order-preserving 32-bit key of a score: larger score, larger key; -0 and +0 equal.
__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace csa
