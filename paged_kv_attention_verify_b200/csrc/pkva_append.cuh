// Fused paged-KV append: writing the new tokens' K/V into their cache slots inside the
// attention launch.
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

// ---- FP8 (E4M3) caches -------------------------------------------------------------------
// A new value's code is E4M3(float32(x) / scale), the division correctly rounded, the
// conversion to nearest even and saturating (every writer below uses this one function,
// so the shared-memory copy the attention reads and the cache agree bit for bit).

// Codes of four consecutive bf16 values, byte i for value i.
__device__ __forceinline__ uint32_t quant4_e4m3(const __nv_bfloat16* src, float scale) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
    float x0, x1, x2, x3;
    bf16x2_to_f32(raw.x, x0, x1);
    bf16x2_to_f32(raw.y, x2, x3);
    const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale));
    const uint32_t hi = f32x2_to_e4m3x2(__fdiv_rn(x2, scale), __fdiv_rn(x3, scale));
    return lo | (hi << 16);
}

// As patch_page_rows, for an FP8 page: the K page (16 rows of D codes, 128- or 64-byte
// swizzle) and the transposed V page (D rows of 16 key bytes) get the new rows' codes.
template <int D>
__device__ __forceinline__ void patch_page_rows_fp8(uint8_t* Kp, uint8_t* Vp, const __nv_bfloat16* k_new,
                                                    const __nv_bfloat16* v_new, const SeqInfo& si, int Hkv,
                                                    int kvh, int r_begin, int r_end, int t0, int lane, float ks,
                                                    float vs) {
    const int rows = r_end - r_begin;
    // K: 16 codes (one 16-byte chunk) per item
    for (int i = lane; i < rows * (D / 16); i += 32) {
        const int r = r_begin + i / (D / 16), c = i % (D / 16);
        const __nv_bfloat16* src = k_new + ((int64_t)(si.q_start + t0 + r - r_begin) * Hkv + kvh) * D + c * 16;
        const uint4 v = make_uint4(quant4_e4m3(src, ks), quant4_e4m3(src + 4, ks), quant4_e4m3(src + 8, ks),
                                   quant4_e4m3(src + 12, ks));
        const int sw = D == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
        *reinterpret_cast<uint4*>(Kp + r * D + (sw << 4)) = v;
    }
    // V: four head-dim rows per item, one byte (key r) in each
    for (int i = lane; i < rows * (D / 4); i += 32) {
        const int r = r_begin + i / (D / 4), d = (i % (D / 4)) * 4;
        const uint32_t q = quant4_e4m3(v_new + ((int64_t)(si.q_start + t0 + r - r_begin) * Hkv + kvh) * D + d, vs);
#pragma unroll
        for (int e = 0; e < 4; ++e) Vp[(d + e) * kPageSize + r] = (uint8_t)(q >> (8 * e));
    }
}

// As append_rows, into FP8 caches: k_cache [pages, Hkv, 16, D] codes, v_cache_t
// [pages, Hkv, D, 16] codes.
template <int D>
__device__ __forceinline__ void append_rows_fp8(const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                                                uint8_t* k_cache, uint8_t* v_cache_t, const int32_t* block_table,
                                                int bt_stride, int num_pages, int Hkv, int* err, const SeqInfo& si,
                                                int seq, int kvh, int t_begin, int t_end, int tid, int n, float ks,
                                                float vs) {
    const int rows = t_end - t_begin;
    if (rows <= 0) return;
    const int prefix = si.seq_len - si.query_len;
    const int32_t* btrow = block_table + (int64_t)seq * bt_stride;
    for (int i = tid; i < rows * (D / 16 + D / 4); i += n) {
        const int t = t_begin + i / (D / 16 + D / 4), j = i % (D / 16 + D / 4);
        const int pos = prefix + t;
        const int page = btrow[pos / kPageSize];
        if (page < 0 || page >= num_pages) {
            atomicOr(err, PKVA_DEVERR_BAD_PAGE);
            continue;
        }
        const int64_t blk = (int64_t)page * Hkv + kvh;
        const int64_t src_row = ((int64_t)(si.q_start + t) * Hkv + kvh) * D;
        if (j < D / 16) {                       // 16 K codes
            const __nv_bfloat16* src = k_new + src_row + j * 16;
            *reinterpret_cast<uint4*>(k_cache + (blk * kPageSize + pos % kPageSize) * D + j * 16) =
                make_uint4(quant4_e4m3(src, ks), quant4_e4m3(src + 4, ks), quant4_e4m3(src + 8, ks),
                           quant4_e4m3(src + 12, ks));
        } else {                                // 4 V codes, one per head-dim row
            const int d = (j - D / 16) * 4;
            const uint32_t q = quant4_e4m3(v_new + src_row + d, vs);
#pragma unroll
            for (int e = 0; e < 4; ++e) v_cache_t[(blk * D + d + e) * kPageSize + pos % kPageSize] = (uint8_t)(q >> (8 * e));
        }
    }
}

}  // namespace pkva
