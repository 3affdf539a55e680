// Split-KV combine shared by the decode/verify tasks and the shared-prefix (cascade) tasks:
// whichever task finishes a unit last merges its partial results into the output rows.
//
// A partial is the unnormalised output O_k, the reference max m_k (log2 units) and the sum
// l_k of one contiguous key range; the full row is sum_k 2^(m_k - M) O_k divided by
// sum_k 2^(m_k - M) l_k with M = max_k m_k (the log-sum-exp merge of FlashAttention-style
// tiling; XY-Serve verdict page, supporting_citations[1]).
//
// The merge is latency-bound (a few partials per row, each read once from L2), so a warp
// merges four rows at once and issues the loads of several partials before using them.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "pkva_internal.h"

namespace pkva {

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Merge the rows of n_units units: unit i is units[uid[i]] and its rows are flattened rows
// [pref[i], pref[i] + its row count) of `total` (uid and pref may live in shared memory).
// Warp `wid` of `nwarps` takes four rows at a time: lane l merges columns
// [(l % 8) * D/8, +D/8) of row l / 8, so each lane has the partials of several slots in
// flight at once.
template <int D>
__device__ __forceinline__ void merge_units(int wid, int nwarps, int lane, const int32_t* uid, const int* pref,
                                            int n_units, int total, const SplitUnit* units, const float* part_o,
                                            const float* part_ml, const SeqInfo* seqs, __nv_bfloat16* out,
                                            int Hq, int G) {
    constexpr int V = D / 8;                            // columns per lane
    constexpr int NQ = V / 4;                           // float4 per lane per slot
    for (int base = wid * 4; base < total; base += nwarps * 4) {
        const int fr = base + (lane >> 3);
        if (fr >= total) continue;
        int lo = 0, hi = n_units - 1;                   // last unit with pref <= fr
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pref[mid] <= fr) lo = mid; else hi = mid - 1;
        }
        const SplitUnit u = units[uid[lo]];
        const int r = fr - pref[lo];
        const int NS = u.num_splits;
        const int col = (lane & 7) * V;
        const int64_t row0 = (int64_t)u.slot_base * kDecodeRowsMax + r;    // slot s: row0 + s * 16
        float M = -INFINITY;
        for (int s0 = 0; s0 < NS; s0 += 8) {
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                m8[k] = s0 + k < NS ? __ldcg(part_ml + (row0 + (int64_t)(s0 + k) * kDecodeRowsMax) * 2) : -INFINITY;
#pragma unroll
            for (int k = 0; k < 8; ++k) M = fmaxf(M, m8[k]);
        }
        float acc[V], L = 0.f;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        if (M != -INFINITY) {
            for (int s0 = 0; s0 < NS; s0 += 2) {
                float2 ml[2];
                float4 o[2][NQ];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int64_t row = row0 + (int64_t)(s0 + k) * kDecodeRowsMax;
                    const bool in = s0 + k < NS;
                    ml[k] = in ? __ldcg(reinterpret_cast<const float2*>(part_ml + row * 2))
                               : make_float2(-INFINITY, 0.f);
#pragma unroll
                    for (int j = 0; j < NQ; ++j)
                        o[k][j] = in ? __ldcg(reinterpret_cast<const float4*>(part_o + row * D + col) + j)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float f = ml[k].x == -INFINITY ? 0.f : exp2f(ml[k].x - M);
                    L = fmaf(f, ml[k].y, L);
#pragma unroll
                    for (int j = 0; j < NQ; ++j) {
                        acc[4 * j] = fmaf(f, o[k][j].x, acc[4 * j]);
                        acc[4 * j + 1] = fmaf(f, o[k][j].y, acc[4 * j + 1]);
                        acc[4 * j + 2] = fmaf(f, o[k][j].z, acc[4 * j + 2]);
                        acc[4 * j + 3] = fmaf(f, o[k][j].w, acc[4 * j + 3]);
                    }
                }
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const int pr = u.row_begin + r;                  // packed row = token * G + head-in-group
        const int t = pr / G;
        const int64_t orow = (int64_t)(seqs[u.seq].q_start + t) * Hq + u.kv_head * G + (pr - t * G);
        uint4* dst = reinterpret_cast<uint4*>(out + orow * D + col);
#pragma unroll
        for (int j = 0; j < V / 8; ++j) {
            uint4 w;
            w.x = pack2(acc[8 * j] * inv, acc[8 * j + 1] * inv);
            w.y = pack2(acc[8 * j + 2] * inv, acc[8 * j + 3] * inv);
            w.z = pack2(acc[8 * j + 4] * inv, acc[8 * j + 5] * inv);
            w.w = pack2(acc[8 * j + 6] * inv, acc[8 * j + 7] * inv);
            dst[j] = w;
        }
    }
}

}  // namespace pkva
