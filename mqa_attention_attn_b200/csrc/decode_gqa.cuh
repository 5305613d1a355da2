// decode_gqa.cuh -- single-token GQA decode against a KV cache, split-KV.
//
// One CTA owns (sequence b, KV head g, a block of GT query heads of that
// group, one chunk of CH consecutive cached keys). The chunk's keys and
// values are streamed HBM -> shared memory by TMA (tile = 64 keys x 128
// dims, 128-byte swizzle) through a 4-stage ring fed by a producer warp; four
// compute warps consume it on the CUDA cores (fp32, packed FFMA2):
//   phase A  scores s[key][h] = <q_h, k_key> * scale * log2(e), all chunk keys
//   phase B  per head: m = max over the chunk, p = 2^(s - m), l = sum p
//   phase C  o[h][:] = sum_key p[key][h] * v_key[:]
// and the partial (o, m, l) goes to the workspace. A second kernel merges the
// chunks of each (b, h) by their log-sum-exp weights.
//
// Each K/V tile is read from HBM once and used by all GT heads of the group
// (the grouped broadcast of "Attention Engineering: From MHA to GQA, MLA &
// FlashAttention", section 2, done in registers); the chunk merge is the
// online-softmax rescaling of section 4 applied across chunks instead of
// tiles. Decode arithmetic intensity is about n_q / n_kv FLOPs per byte
// (same page, section 0), so this kernel is bound by HBM bandwidth: the
// design goal is to keep the ring full and the CUDA-core work per byte small.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace dec {

constexpr int D = 128;            // head dim (keys and values)
constexpr int KT = 64;            // keys per tile
constexpr int CH = 512;           // keys per chunk (one CTA)
constexpr int NSTAGE = 4;         // ring depth
constexpr int TILE_BYTES = KT * D * 2;      // 16 KB: two 64-dim boxes of 64 rows x 128 B
constexpr int BOX_BYTES = KT * 128;         // one 64-dim box
constexpr int NCW = 4;            // compute warps
constexpr int THREADS = (NCW + 1) * 32;

template <int GT>
struct Smem {
    uint8_t ring[NSTAGE][TILE_BYTES];       // 1024-byte aligned (swizzle atoms)
    float scores[CH * GT];                  // [key][head], log2 units, then p
    float opart[NCW][GT][D];                // per-warp partial outputs
    float red_m[NCW][GT];
    float red_l[NCW][GT];
    uint64_t full[NSTAGE];
    uint64_t empty[NSTAGE];
    int abort_flag;
};

template <int GT>
constexpr size_t smem_bytes() {
    return sizeof(Smem<GT>) + 1024;  // + alignment slack
}

// Mapping of compute warps in phase A: each thread holds a quarter of the
// head dim (32 values) of HPT heads; warps split into HS head sets x KS key
// sets.
template <int GT>
struct QkMap {
    static constexpr int HPT = GT < 2 ? GT : 2;
    static constexpr int HS = GT / HPT;
    static constexpr int KS = NCW / HS;
    static_assert(HS * KS == NCW, "head block must map onto 4 warps");
};

template <int GT>
__global__ void __launch_bounds__(THREADS, 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16 *__restrict__ q, const int32_t *__restrict__ seqlens,
                    float *__restrict__ ws_o, float2 *__restrict__ ws_ml, int n_q, int G, int n_hb,
                    int S_max, int n_splits, float scale_log2) {
    using Map = QkMap<GT>;
    extern __shared__ uint8_t smem_raw[];
    Smem<GT> &sm = *reinterpret_cast<Smem<GT> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int split = blockIdx.x;
    const int kvh = blockIdx.y / n_hb;
    const int hb = blockIdx.y % n_hb;
    const int b = blockIdx.z;
    int seqlen = seqlens[b];
    if (seqlen > S_max) {
        if (threadIdx.x == 0 && split == 0 && blockIdx.y == 0) atomicOr(&g_status, kStatusRange);
        seqlen = S_max;
    }
    if (seqlen < 0) seqlen = 0;
    const int key0 = split * CH;
    if (key0 >= seqlen) return;  // uniform for the CTA
    const int nkeys = min(CH, seqlen - key0);
    const int ntiles = (nkeys + KT - 1) / KT;
    const int h0 = kvh * G + hb * GT;  // first query head of this CTA

    const uint32_t warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), NCW);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int *abort_flag = &sm.abort_flag;

    if (warp == NCW) {
        // ---------------- producer warp ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int issued = 0;
            for (int t = 0; t < 2 * ntiles; ++t) {
                const int s = t % NSTAGE;
                const uint32_t ph = (t / NSTAGE) & 1;
                if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1, abort_flag, 0x101)) break;
                const uint32_t full = smem_u32(&sm.full[s]);
                mbar_arrive_expect_tx(full, TILE_BYTES);
                const CUtensorMap *tm = (t < ntiles) ? &tm_k : &tm_v;
                const int krow = key0 + (t < ntiles ? t : t - ntiles) * KT;
                const uint32_t dst = smem_u32(sm.ring[s]);
                tma_load_4d(dst, tm, full, 0, krow, kvh, b);
                tma_load_4d(dst + BOX_BYTES, tm, full, 64, krow, kvh, b);
                ++issued;
            }
            // Do not leave while copies into this CTA's shared memory are in
            // flight: wait (bounded) for the last issued tile of each stage.
            for (int t = issued - 1; t >= 0 && t >= issued - NSTAGE; --t)
                mbar_wait(smem_u32(&sm.full[t % NSTAGE]), (t / NSTAGE) & 1, nullptr, 0x102);
        }
        return;
    }

    // ---------------- compute warps (128 threads) ----------------
    const int tid = threadIdx.x;  // 0..127

    // phase A: scores ------------------------------------------------------
    {
        const int hs = warp / Map::KS;        // head set
        const int ks = warp % Map::KS;        // key set
        const int quarter = lane >> 3;        // which 32 dims
        const int kl = lane & 7;              // key within the warp's 8
        float2 qr[Map::HPT][16];
#pragma unroll
        for (int hh = 0; hh < Map::HPT; ++hh) {
            const int h = h0 + hs * Map::HPT + hh;
            const uint4 *src = reinterpret_cast<const uint4 *>(q + ((size_t)b * n_q + h) * D + quarter * 32);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 w = __ldg(src + c);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 f = bf2_to_f2(ws[e]);
                    qr[hh][c * 4 + e] = make_float2(f.x * scale_log2, f.y * scale_log2);
                }
            }
        }
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % NSTAGE;
            if (!mbar_wait(smem_u32(&sm.full[s]), (t / NSTAGE) & 1, abort_flag, 0x201)) break;
            const uint32_t base = smem_u32(sm.ring[s]);
#pragma unroll 2
            for (int p = 0; p < KT / (8 * Map::KS); ++p) {
                const int key = p * 8 * Map::KS + ks * 8 + kl;  // key within the tile
                float2 acc[Map::HPT];
#pragma unroll
                for (int hh = 0; hh < Map::HPT; ++hh) acc[hh] = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = quarter * 4 + i;  // 16-byte chunk of the 256-byte row
                    const uint32_t off = (uint32_t)((c >> 3) * BOX_BYTES) + swz<3>((uint32_t)(key * 128 + (c & 7) * 16));
                    const uint4 w = lds128(base + off);
                    const float2 k0 = bf2_to_f2(w.x), k1 = bf2_to_f2(w.y), k2 = bf2_to_f2(w.z), k3 = bf2_to_f2(w.w);
#pragma unroll
                    for (int hh = 0; hh < Map::HPT; ++hh) {
                        acc[hh] = ffma2(qr[hh][i * 4 + 0], k0, acc[hh]);
                        acc[hh] = ffma2(qr[hh][i * 4 + 1], k1, acc[hh]);
                        acc[hh] = ffma2(qr[hh][i * 4 + 2], k2, acc[hh]);
                        acc[hh] = ffma2(qr[hh][i * 4 + 3], k3, acc[hh]);
                    }
                }
#pragma unroll
                for (int hh = 0; hh < Map::HPT; ++hh) {
                    float sc = acc[hh].x + acc[hh].y;
                    sc += __shfl_xor_sync(0xffffffffu, sc, 8);
                    sc += __shfl_xor_sync(0xffffffffu, sc, 16);
                    if (quarter == hh) sm.scores[(t * KT + key) * GT + hs * Map::HPT + hh] = sc;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
        }
    }
    if (named_bar_or(1, NCW * 32, *abort_flag != 0)) return;

    // phase B: softmax statistics over the chunk ------------------------------
    float m[GT], l[GT];
    {
        float mloc[GT];
#pragma unroll
        for (int h = 0; h < GT; ++h) mloc[h] = -INFINITY;
        for (int key = tid; key < nkeys; key += NCW * 32) {
#pragma unroll
            for (int h = 0; h < GT; ++h) mloc[h] = fmaxf(mloc[h], sm.scores[key * GT + h]);
        }
#pragma unroll
        for (int h = 0; h < GT; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mloc[h] = fmaxf(mloc[h], __shfl_xor_sync(0xffffffffu, mloc[h], o));
            if (lane == 0) sm.red_m[warp][h] = mloc[h];
        }
        named_bar_sync(1, NCW * 32);
#pragma unroll
        for (int h = 0; h < GT; ++h) {
            m[h] = sm.red_m[0][h];
#pragma unroll
            for (int w = 1; w < NCW; ++w) m[h] = fmaxf(m[h], sm.red_m[w][h]);
        }
        float lloc[GT];
#pragma unroll
        for (int h = 0; h < GT; ++h) lloc[h] = 0.f;
        for (int key = tid; key < ntiles * KT; key += NCW * 32) {
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                float pv = 0.f;
                if (key < nkeys) pv = ex2(sm.scores[key * GT + h] - m[h]);
                sm.scores[key * GT + h] = pv;
                lloc[h] += pv;
            }
        }
#pragma unroll
        for (int h = 0; h < GT; ++h) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lloc[h] += __shfl_xor_sync(0xffffffffu, lloc[h], o);
            if (lane == 0) sm.red_l[warp][h] = lloc[h];
        }
        named_bar_sync(1, NCW * 32);
#pragma unroll
        for (int h = 0; h < GT; ++h) {
            l[h] = 0.f;
#pragma unroll
            for (int w = 0; w < NCW; ++w) l[h] += sm.red_l[w][h];
        }
    }

    // phase C: p . V ------------------------------------------------------------
    float2 oacc[GT][2];
#pragma unroll
    for (int h = 0; h < GT; ++h) oacc[h][0] = oacc[h][1] = make_float2(0.f, 0.f);
    {
        const int c = lane >> 1;       // 16-byte chunk holding this lane's 4 dims
        const int half = lane & 1;
        const uint32_t box_off = (uint32_t)((c >> 3) * BOX_BYTES);
        for (int t = 0; t < ntiles; ++t) {
            const int tt = ntiles + t;
            const int s = tt % NSTAGE;
            if (!mbar_wait(smem_u32(&sm.full[s]), (tt / NSTAGE) & 1, abort_flag, 0x301)) break;
            const uint32_t base = smem_u32(sm.ring[s]) + box_off;
            const float *ps = sm.scores + (size_t)t * KT * GT;
#pragma unroll 4
            for (int kk = warp; kk < KT; kk += NCW) {
                const uint2 w = lds64(base + swz<3>((uint32_t)(kk * 128 + (c & 7) * 16)) + half * 8);
                const float2 v0 = bf2_to_f2(w.x), v1 = bf2_to_f2(w.y);
                float pk[GT];
                if constexpr (GT % 4 == 0) {
#pragma unroll
                    for (int h4 = 0; h4 < GT / 4; ++h4) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(ps + kk * GT + h4 * 4);
                        pk[h4 * 4 + 0] = t4.x;
                        pk[h4 * 4 + 1] = t4.y;
                        pk[h4 * 4 + 2] = t4.z;
                        pk[h4 * 4 + 3] = t4.w;
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < GT; ++h) pk[h] = ps[kk * GT + h];
                }
#pragma unroll
                for (int h = 0; h < GT; ++h) {
                    const float2 pp = make_float2(pk[h], pk[h]);
                    oacc[h][0] = ffma2(pp, v0, oacc[h][0]);
                    oacc[h][1] = ffma2(pp, v1, oacc[h][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
        }
    }
    // combine the four warps' partial sums, write (o, m, l) of this chunk
#pragma unroll
    for (int h = 0; h < GT; ++h)
        *reinterpret_cast<float4 *>(&sm.opart[warp][h][lane * 4]) =
            make_float4(oacc[h][0].x, oacc[h][0].y, oacc[h][1].x, oacc[h][1].y);
    if (named_bar_or(1, NCW * 32, *abort_flag != 0)) return;
#pragma unroll
    for (int j = 0; j < GT; ++j) {
        const int idx = tid + j * NCW * 32;  // over GT * D outputs
        const int h = idx / D, d = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) acc += sm.opart[w][h][d];
        ws_o[(((size_t)b * n_q + h0 + h) * n_splits + split) * D + d] = acc;
    }
    if (tid < GT) ws_ml[((size_t)b * n_q + h0 + tid) * n_splits + split] = make_float2(m[tid], l[tid]);
}

// Merge the chunks of each (b, h): M = max m_s, w_s = 2^(m_s - M),
// O = sum w_s o_s / sum w_s l_s, LSE = (M + log2 sum w_s l_s) * ln 2.
// One CTA per (h, b); thread i owns output dims i, i + blockDim, ...
__global__ void __launch_bounds__(128)
decode_combine_kernel(const float *__restrict__ ws_o, const float2 *__restrict__ ws_ml,
                      const int32_t *__restrict__ seqlens, __nv_bfloat16 *__restrict__ o,
                      float *__restrict__ lse, int n_q, int n_splits, int S_max, int chunk, int d_v) {
    const int h = blockIdx.x, b = blockIdx.y;
    int seqlen = seqlens[b];
    seqlen = seqlen < 0 ? 0 : (seqlen > S_max ? S_max : seqlen);
    const int ns = (seqlen + chunk - 1) / chunk;
    const size_t row = (size_t)b * n_q + h;
    const float2 *ml = ws_ml + row * n_splits;
    if (ns == 0) {
        for (int d = threadIdx.x; d < d_v; d += blockDim.x) o[row * d_v + d] = __float2bfloat16_rn(0.f);
        if (threadIdx.x == 0 && lse) lse[row] = -INFINITY;
        return;
    }
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[s].x);
    float L = 0.f;
    for (int s = 0; s < ns; ++s) L += ex2(ml[s].x - M) * ml[s].y;
    const float inv = 1.f / L;
    for (int d = threadIdx.x; d < d_v; d += blockDim.x) {
        float acc = 0.f;
        for (int s = 0; s < ns; ++s) acc += ex2(ml[s].x - M) * ws_o[(row * n_splits + s) * d_v + d];
        o[row * d_v + d] = __float2bfloat16_rn(acc * inv);
    }
    if (threadIdx.x == 0 && lse) lse[row] = (M + log2f(L)) * 0.6931471805599453f;
}

}  // namespace dec
}  // namespace attn
