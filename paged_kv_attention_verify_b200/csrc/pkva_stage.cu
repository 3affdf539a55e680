// FP8 (E4M3) caches on the tensor-core path: bf16 staging copies of the code pages that the
// tensor-core (prefill) tasks read. tcgen05 multiplies bf16 tiles, and every E4M3 value is
// a bf16 value, so the copy is exact and unscaled: the tasks fold the K scale of their KV
// head into the softmax scale and the V scale into the output. One block per staging page
// does all KV heads of that page; slots past the sequence's end are staged as zeros (their
// codes may be NaN). With the fused append, the new tokens' codes are computed here from
// k_new / v_new (the same rounding as every other writer), stored into the FP8 caches and
// staged, so the attention launch that follows reads exactly what the caches now hold.
//
// Sources: XY-Serve (arXiv 2412.18106), verdict page — the quantized KV formats the pages
// name; chunked prefill on cached prefixes (core_discovery).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pkva.h"
#include "pkva_append.cuh"
#include "pkva_kernels.h"
#include "pkva_ptx.cuh"

namespace pkva {
namespace {

constexpr int kD = 128;                 // tensor-core tasks run at head_dim 128 only
constexpr int kStageThreads = 256;

// Four codes (byte 0 first) to four bf16 in two words (value 0 in the low half of .x).
__device__ __forceinline__ uint2 e4m3x4_to_bf16x4(uint32_t codes) {
    uint32_t lo, hi;
    e4m3x4_to_f16x2x2(codes, lo, hi);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    return make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y));
}

__global__ void __launch_bounds__(kStageThreads) stage_fp8_kernel(const StageParams p) {
    __shared__ __align__(16) uint8_t vt[kD * kPageSize];     // one transposed V page block
    const int n = blockIdx.x, tid = threadIdx.x;
    const int seq = p.src[2 * n], lp = p.src[2 * n + 1];
    const SeqInfo si = p.seqs[seq];
    const int prefix = si.seq_len - si.query_len;
    const int key0 = lp * kPageSize;                          // the page's first key
    int ph = p.block_table[(int64_t)seq * p.bt_stride + lp];
    if (ph < 0 || ph >= p.num_pages) {
        if (tid == 0) atomicOr(p.err, PKVA_DEVERR_BAD_PAGE);
        ph = -1;                                              // staged as zeros
    }
    // new tokens in this page: slots [r_lo, r_hi)
    const int r_lo = max(prefix - key0, 0), r_hi = min(si.seq_len - key0, kPageSize);
    const bool appends = p.append && ph >= 0 && r_hi > r_lo;

    for (int h = 0; h < p.Hkv; ++h) {
        const int64_t blk = (int64_t)ph * p.Hkv + h;          // (page, head) block of the caches
        const int64_t sblk = (int64_t)n * p.Hkv + h;          // (staging page, head) block
        if (tid < 128) {
            // K: row r, codes 16c .. 16c+15 -> 16 bf16
            const int r = tid >> 3, c = tid & 7;
            const bool valid = ph >= 0 && key0 + r < si.seq_len;
            uint4 codes = make_uint4(0u, 0u, 0u, 0u);
            if (valid) {
                uint8_t* cache = p.k_codes + (blk * kPageSize + r) * kD + c * 16;
                if (appends && r >= r_lo) {
                    const __nv_bfloat16* src =
                        p.k_new + ((int64_t)(si.q_start + key0 + r - prefix) * p.Hkv + h) * kD + c * 16;
                    const float ks = p.k_scale[h];
                    codes = make_uint4(quant4_e4m3(src, ks), quant4_e4m3(src + 4, ks), quant4_e4m3(src + 8, ks),
                                       quant4_e4m3(src + 12, ks));
                    *reinterpret_cast<uint4*>(cache) = codes;
                } else {
                    codes = *reinterpret_cast<const uint4*>(cache);
                }
            }
            uint4 o0 = make_uint4(0u, 0u, 0u, 0u), o1 = o0;
            if (valid) {
                const uint2 a = e4m3x4_to_bf16x4(codes.x), b = e4m3x4_to_bf16x4(codes.y);
                const uint2 c2 = e4m3x4_to_bf16x4(codes.z), d = e4m3x4_to_bf16x4(codes.w);
                o0 = make_uint4(a.x, a.y, b.x, b.y);
                o1 = make_uint4(c2.x, c2.y, d.x, d.y);
            }
            uint4* out = reinterpret_cast<uint4*>(p.stage_k + (sblk * kPageSize + r) * kD + c * 16);
            out[0] = o0;
            out[1] = o1;
        } else {
            // V^T: head-dim row i of the page block (16 key bytes) into shared memory
            const int i = tid - 128;
            uint4 row = make_uint4(0u, 0u, 0u, 0u);
            if (ph >= 0) row = *reinterpret_cast<const uint4*>(p.v_codes_t + (blk * kD + i) * kPageSize);
            *reinterpret_cast<uint4*>(vt + i * kPageSize) = row;
        }
        __syncthreads();
        if (appends) {
            // the new tokens' V codes: key slot r, four head-dim rows per item
            for (int i = tid; i < (r_hi - r_lo) * (kD / 4); i += kStageThreads) {
                const int r = r_lo + i / (kD / 4), d = (i % (kD / 4)) * 4;
                const uint32_t q =
                    quant4_e4m3(p.v_new + ((int64_t)(si.q_start + key0 + r - prefix) * p.Hkv + h) * kD + d,
                                p.v_scale[h]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint8_t b = (uint8_t)(q >> (8 * e));
                    vt[(d + e) * kPageSize + r] = b;
                    p.v_codes_t[(blk * kD + d + e) * kPageSize + r] = b;
                }
            }
            __syncthreads();
        }
        {
            // V: key r, head-dim columns 8c .. 8c+7 -> one 16-byte chunk of bf16
            const int r = tid >> 4, c = tid & 15;
            uint4 o = make_uint4(0u, 0u, 0u, 0u);
            if (ph >= 0 && key0 + r < si.seq_len) {
                uint32_t lo = 0u, hi = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    lo |= (uint32_t)vt[(8 * c + e) * kPageSize + r] << (8 * e);
                    hi |= (uint32_t)vt[(8 * c + 4 + e) * kPageSize + r] << (8 * e);
                }
                const uint2 a = e4m3x4_to_bf16x4(lo), b = e4m3x4_to_bf16x4(hi);
                o = make_uint4(a.x, a.y, b.x, b.y);
            }
            *reinterpret_cast<uint4*>(p.stage_v + (sblk * kPageSize + r) * kD + c * 8) = o;
        }
        __syncthreads();                                      // vt is refilled for the next head
    }
}

}  // namespace

cudaError_t launch_stage_fp8(const StageParams& p, cudaStream_t stream) {
    if (p.n <= 0) return cudaSuccess;
    stage_fp8_kernel<<<p.n, kStageThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pkva
