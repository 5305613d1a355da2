// rope.cuh -- rotary position embedding for the attention kernels (sm_100a).
//
// "Attention Engineering: From MHA to GQA, MLA & FlashAttention", section 1
// (Rotary Position Embeddings): the head dimension d is split into d/2
// planes (x_{2j}, x_{2j+1}); at position m plane j turns by the angle
// m * theta_j, theta_j = base^(-2j/d):
//     x'_{2j}   = x_{2j} cos(m theta_j) - x_{2j+1} sin(m theta_j)
//     x'_{2j+1} = x_{2j} sin(m theta_j) + x_{2j+1} cos(m theta_j)
// Section 2 applies it to the queries and the keys before the scores.
//
// The angles come from fp32 tables cos/sin [n_pos][d/2] (the cache tables
// of section 1). Here:
//   * rope_tables_kernel fills them (angles in fp64, rounded once to fp32);
//   * rope_apply_kernel rotates a bf16 [rows][d] tensor in global memory
//     (one pass, bandwidth-bound; used for keys, which many query tiles read);
//   * rope_chunk rotates 8 bf16 values (4 planes) held in a 16-byte word, the
//     step the attention kernels apply to Q tiles in shared memory.
// The rotation runs in fp32 (one product and one fused multiply-add per
// output) and is rounded to bf16 once.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace rope {

struct Tables {
    const float *cos;   // [n_pos][d/2]; null: no rotation
    const float *sin;
    int n_pos;
};

// Rotate the 4 planes of one 16-byte word of bf16 pairs; c, s: the 4 angles.
__device__ __forceinline__ uint4 rope_chunk(uint4 w, float4 c, float4 s) {
    auto rot = [](uint32_t x, float cc, float ss) -> uint32_t {
        const float2 f = bf2_to_f2(x);   // f.x = x_{2j}, f.y = x_{2j+1}
        return f2_to_bf2(fmaf(f.x, cc, -(f.y * ss)), fmaf(f.x, ss, f.y * cc));
    };
    w.x = rot(w.x, c.x, s.x);
    w.y = rot(w.y, c.y, s.y);
    w.z = rot(w.z, c.z, s.z);
    w.w = rot(w.w, c.w, s.w);
    return w;
}

// A 128-row tile of D dims, TMA-loaded and swizzled in shared memory (boxes
// of ROWB bytes per row -- 128: SW128, 64: SW64, 32: SW32 -- `box_bytes`
// apart), rotated in place by 128 threads. Thread t takes the 16-byte words
// g = it * 128 + t (it < D/8): word g % (D/8) of row g / (D/8), so that the
// lanes of a warp read whole table rows (coalesced) and each 8-lane phase of
// a shared access hits 8 distinct bank groups. The angles are fetched first
// (fetch(), before the tile has arrived, so that their latency overlaps the
// tile's load), then applied (apply()). `apos(row)` gives a row's table
// position, `valid(row)` whether it holds data.
template <int D, int ROWB>
struct RopeTile {
    static constexpr int SWB = ROWB == 128 ? 3 : (ROWB == 64 ? 2 : 1);
    static constexpr int NW = D / 8;                 // 16-byte words of a row (4 planes each)
    static constexpr int CPR = ROWB / 16;            // words per box row
    float4 c[NW], s[NW];
    template <class PosFn>
    __device__ __forceinline__ void fetch(const Tables &t, int tid, PosFn apos) {
#pragma unroll
        for (int it = 0; it < NW; ++it) {
            const int g = it * 128 + tid, row = g / NW, w = g % NW;
            const size_t off = (size_t)apos(row) * (D / 2) + (size_t)w * 4;
            c[it] = __ldg(reinterpret_cast<const float4 *>(t.cos + off));
            s[it] = __ldg(reinterpret_cast<const float4 *>(t.sin + off));
        }
    }
    template <class ValidFn>
    __device__ __forceinline__ void apply(uint32_t tile, uint32_t box_bytes, int tid, ValidFn valid) const {
#pragma unroll
        for (int it = 0; it < NW; ++it) {
            const int g = it * 128 + tid, row = g / NW, w = g % NW;
            if (!valid(row)) continue;
            const uint32_t a = tile + (uint32_t)(w / CPR) * box_bytes +
                               swz<SWB>((uint32_t)(row * ROWB + (w % CPR) * 16));
            sts128(a, rope_chunk(lds128(a), c[it], s[it]));
        }
    }
};

// cos/sin [n_pos][half]: angle m * base^(-2j/d) in fp64, rounded to fp32.
__global__ void rope_tables_kernel(float *cos_t, float *sin_t, int n_pos, int half, double base) {
    const long long n = (long long)n_pos * half;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / half), j = (int)(i % half);
        const double theta = pow(base, -(double)j / (double)half);   // = base^(-2j/d)
        double sv, cv;
        sincos((double)m * theta, &sv, &cv);
        cos_t[i] = (float)cv;
        sin_t[i] = (float)sv;
    }
}

// y[bh][s] = x[bh][s] rotated at position pos0 + s: rows of d bf16 values,
// [BH][S][d] contiguous (x and y may be the same buffer). Grid: x over the
// 16-byte words of S rows (32-bit index), y over groups of ROPE_BH row blocks
// (strided): a thread fetches its word's angles once and rotates that word in
// ROPE_BH row blocks, all loads issued before the stores.
constexpr int ROPE_BH = 4;
__global__ void rope_apply_kernel(const __nv_bfloat16 *x, __nv_bfloat16 *y, long long BH, int S, int d, int pos0,
                                  Tables t) {
    griddep_launch_dependents();                 // the attention kernel may start its prologue
    const int cpr = d / 8;                       // words per row
    const int w = blockIdx.x * blockDim.x + threadIdx.x;
    if (w >= S * cpr) return;
    const int srow = w / cpr, c = w - srow * cpr;
    int pos = pos0 + srow;
    if (pos >= t.n_pos) {
        atomicOr(&g_status, kStatusRange);
        pos = t.n_pos - 1;
    }
    const size_t tab = (size_t)pos * (d / 2) + (size_t)c * 4;
    const float4 cc = __ldg(reinterpret_cast<const float4 *>(t.cos + tab));
    const float4 ss = __ldg(reinterpret_cast<const float4 *>(t.sin + tab));
    const size_t plane = (size_t)S * cpr;        // words of one row block
    for (long long bh0 = (long long)blockIdx.y * ROPE_BH; bh0 < BH; bh0 += (long long)gridDim.y * ROPE_BH) {
        uint4 v[ROPE_BH];
#pragma unroll
        for (int k = 0; k < ROPE_BH; ++k)
            if (bh0 + k < BH) v[k] = __ldg(reinterpret_cast<const uint4 *>(x) + (size_t)(bh0 + k) * plane + w);
#pragma unroll
        for (int k = 0; k < ROPE_BH; ++k)
            if (bh0 + k < BH) reinterpret_cast<uint4 *>(y)[(size_t)(bh0 + k) * plane + w] = rope_chunk(v[k], cc, ss);
    }
}

}  // namespace rope
}  // namespace attn
