// Fused paged-KV append: writing the new tokens' K/V into their cache slots inside the
// attention launch (survey section 8, next row 1).
//
// Attention tasks never read these writes: a decode/verify task patches the new tokens'
// rows into its shared-memory copy of each page from the dense input, and a prefill task
// loads its chunk's keys from the dense input. So the writes can run beside the reads in
// the same launch; one task per (sequence, KV head) makes them.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "pkva.h"
#include "pkva_internal.h"
#include "pkva_ptx.cuh"

namespace pkva {

// Copy new tokens [t_begin, t_end) of (seq, kvh) from k_new / v_new ([sum T, Hkv, D], q's
// token order) to their cache slots through the block table; threads tid, tid + n, ... of
// the caller each move 16-byte pieces, four loads in flight before their stores. An
// out-of-range page is flagged and skipped.
template <int D>
__device__ __forceinline__ void append_rows(const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                            __nv_bfloat16* k_cache, __nv_bfloat16* v_cache,
                                            const int32_t* block_table, int bt_stride, int num_pages, int Hkv,
                                            int* err, const SeqInfo& si, int seq, int kvh, int t_begin, int t_end,
                                            int tid, int n) {
    constexpr int kPieces = D / 8;                       // 16-byte pieces per row
    constexpr int kBatch = 4;
    const int rows = t_end - t_begin;
    if (rows <= 0) return;
    const int total = 2 * rows * kPieces;
    const int prefix = si.seq_len - si.query_len;
    const int32_t* btrow = block_table + (int64_t)seq * bt_stride;
    for (int i0 = tid; i0 < total; i0 += kBatch * n) {
        uint4 val[kBatch];
        __nv_bfloat16* dst[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int i = i0 + b * n;
            dst[b] = nullptr;
            if (i >= total) continue;
            const int which = i / (rows * kPieces);      // 0: K, 1: V
            const int rem = i - which * rows * kPieces;
            const int t = t_begin + rem / kPieces;
            const int c = rem - (rem / kPieces) * kPieces;
            const int pos = prefix + t;
            const int page = btrow[pos / kPageSize];
            if (page < 0 || page >= num_pages) {
                atomicOr(err, PKVA_DEVERR_BAD_PAGE);
                continue;
            }
            val[b] = __ldg(reinterpret_cast<const uint4*>((which ? v_new : k_new) +
                                                          ((int64_t)(si.q_start + t) * Hkv + kvh) * D + c * 8));
            dst[b] = (which ? v_cache : k_cache) + (((int64_t)page * Hkv + kvh) * kPageSize + pos % kPageSize) * D +
                     c * 8;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
            if (dst[b]) *reinterpret_cast<uint4*>(dst[b]) = val[b];
    }
}

// Overwrite, in a page's shared-memory copy (K and V, 16 rows, 128-byte swizzle, boxes of
// 64 columns), the rows of new tokens with the dense input; the 32 lanes of a warp
// cooperate with register-free 16-byte async copies, then wait for their own. The caller
// syncs the warp before other lanes read the rows. Rows [r_begin, r_end) of the page hold
// new tokens starting at new-token index t0.
template <int D>
__device__ __forceinline__ void patch_page_rows(uint8_t* Ks, uint8_t* Vs, const __nv_bfloat16* k_new,
                                                const __nv_bfloat16* v_new, const SeqInfo& si, int Hkv, int kvh,
                                                int r_begin, int r_end, int t0, int lane) {
    constexpr int kPieces = D / 8;
    constexpr int kBox = kPageSize * 128;
    const int rows = r_end - r_begin;
    for (int i = lane; i < 2 * rows * kPieces; i += 32) {
        const int which = i / (rows * kPieces);
        const int rem = i - which * rows * kPieces;
        const int r = r_begin + rem / kPieces;
        const int c = rem - (rem / kPieces) * kPieces;
        const int t = t0 + (r - r_begin);
        cp_async_16((which ? Vs : Ks) + (c >> 3) * kBox + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                    (which ? v_new : k_new) + ((int64_t)(si.q_start + t) * Hkv + kvh) * D + c * 8);
    }
    cp_async_wait_all();
}

}  // namespace pkva
