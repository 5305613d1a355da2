// e4m3 -> bf16 widening of the FP8 prefill's operands.
//
// Source: "Flash Attention 3 and Multi-Headed Latent Attention", FP8 section
// (e4m3 operands with scaling factors). Every e4m3 value is exactly a bf16
// value (4 significant bits, exponents 2^-9 .. 2^8), so the widened arrays
// carry the same numbers; the scales stay apart and are applied inside the
// attention kernel.
#pragma once

#include <cstddef>
#include <cstdint>

#include "sm100.cuh"

namespace attn {
namespace f8 {

// One array to widen: `n16` groups of 16 e4m3 bytes from src into 16 bf16
// values (32 bytes) each at dst; both 16-byte aligned.
struct WidenSeg {
    const uint8_t *src;
    uint16_t *dst;
    size_t n16;
};

constexpr int WIDEN_THREADS = 256;

constexpr int WIDEN_UNROLL = 4;   // 16-byte loads in flight per thread

// Groups i, i + stride, ... of one array: WIDEN_UNROLL independent loads
// issued before their conversions and stores.
__device__ __forceinline__ void widen_array(const uint8_t *src, uint16_t *dst, size_t n16, size_t first,
                                            size_t stride) {
    const uint4 *in = reinterpret_cast<const uint4 *>(src);
    uint4 *out = reinterpret_cast<uint4 *>(dst);
    for (size_t i = first; i < n16; i += WIDEN_UNROLL * stride) {
        uint4 x[WIDEN_UNROLL];
#pragma unroll
        for (int u = 0; u < WIDEN_UNROLL; ++u) {
            const size_t k = i + u * stride;
            if (k < n16) x[u] = __ldg(in + k);
        }
#pragma unroll
        for (int u = 0; u < WIDEN_UNROLL; ++u) {
            const size_t k = i + u * stride;
            if (k < n16) {
                out[2 * k] = e4m3x8_to_bf16x8(x[u].x, x[u].y);
                out[2 * k + 1] = e4m3x8_to_bf16x8(x[u].z, x[u].w);
            }
        }
    }
}

// The three operands in one launch: a grid-stride pass over each (coalesced
// 16-byte loads, two 16-byte stores per load).
__global__ void __launch_bounds__(WIDEN_THREADS) widen_e4m3_kernel(const WidenSeg a, const WidenSeg b,
                                                                    const WidenSeg c) {
    // the attention grid launched after this one may start its prologue
    // (it waits for this grid before it reads the widened arrays)
    griddep_launch_dependents();
    const size_t first = (size_t)blockIdx.x * WIDEN_THREADS + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * WIDEN_THREADS;
    widen_array(a.src, a.dst, a.n16, first, stride);
    widen_array(b.src, b.dst, b.n16, first, stride);
    widen_array(c.src, c.dst, c.n16, first, stride);
}

}  // namespace f8
}  // namespace attn
