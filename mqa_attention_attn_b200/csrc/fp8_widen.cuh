// e4m3 -> f16 widening of the FP8 prefill's operands.
//
// Source: "Flash Attention 3 and Multi-Headed Latent Attention", FP8 section
// (e4m3 operands with scaling factors). Every e4m3 value is exactly an f16
// value, so the widened arrays carry the same numbers; the scales stay apart
// and are applied inside the attention kernel.
#pragma once

#include <cstddef>
#include <cstdint>

#include "sm100.cuh"

namespace attn {
namespace f8 {

// One array to widen: `n16` groups of 16 e4m3 bytes from src into 16 f16
// values (32 bytes) each at dst; both 16-byte aligned.
struct WidenSeg {
    const uint8_t *src;
    uint16_t *dst;
    size_t n16;
};

constexpr int WIDEN_THREADS = 256;

// The three operands in one launch: a grid-stride loop over the groups of
// a, then b, then c (coalesced 16-byte loads, two 16-byte stores each).
__global__ void __launch_bounds__(WIDEN_THREADS) widen_e4m3_kernel(const WidenSeg a, const WidenSeg b,
                                                                    const WidenSeg c) {
    const size_t nab = a.n16 + b.n16, total = nab + c.n16;
    for (size_t i = (size_t)blockIdx.x * WIDEN_THREADS + threadIdx.x; i < total;
         i += (size_t)gridDim.x * WIDEN_THREADS) {
        const uint8_t *src;
        uint16_t *dst;
        size_t k;
        if (i < a.n16) {
            src = a.src, dst = a.dst, k = i;
        } else if (i < nab) {
            src = b.src, dst = b.dst, k = i - a.n16;
        } else {
            src = c.src, dst = c.dst, k = i - nab;
        }
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src) + k);
        uint4 *d = reinterpret_cast<uint4 *>(dst) + 2 * k;
        d[0] = e4m3x8_to_f16x8(x.x, x.y);
        d[1] = e4m3x8_to_f16x8(x.z, x.w);
    }
}

}  // namespace f8
}  // namespace attn
