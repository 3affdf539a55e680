// Causal chunked-prefill attention over the paged KV cache on 5th-generation tensor cores
// (K-P): S = Q K^T and O += P V are tcgen05.mma BF16 tiles with fp32 accumulators in
// tensor memory (TMEM).
//
// One CTA runs one tile task: 128 query tokens of one query head (tcgen05 M = 128) against
// the 128-key KV tiles (8 pages, gathered by TMA through the block table) that the causal
// mask leaves visible; tiles past the last row's own position are never loaded (causal
// tile skipping), and only tiles that cross the diagonal are masked element by element.
//
// Warp roles (224 threads):
//   warps 0-3  softmax: thread r owns row r = TMEM lane r. Reads S, keeps the running
//              max / sum, writes P (bf16) back to TMEM, rescales O in TMEM only when a
//              row max moved by more than 2^8 (rare after the first tiles), and writes O.
//   warp 4     TMA producer of Q and of K tiles (3-stage ring, a stage is freed as soon as
//              its QK^T is done); warp 6 produces V tiles (2-stage ring, freed after PV).
//   warp 5     MMA issuer (one thread) and TMEM owner: QK^T of tile j+1 overlaps the
//              softmax of tile j; PV of tile j reads P straight from TMEM.
// TMEM (512 columns): S double buffer [0,256), O [256,384), P double buffer [384,512).
//
// Sources: XY-Serve (arXiv 2412.18106), verdict page — key_machinery (the attention
// primitive is a matmul-softmax-matmul tile whose QK and SV products overlap the softmax),
// core_discovery (chunked prefill on cached prefixes; fully masked tiles are skipped);
// supporting citation [1] (FlashAttention's tiled online softmax).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkva.h"
#include "pkva_kernels.h"
#include "pkva_ptx.cuh"

namespace pkva {

namespace {

constexpr int kPThreads = 224;
constexpr int kD = 128;
constexpr int kNK = 3;                                   // K stages (freed when QK^T is done)
constexpr int kNV = 2;                                   // V stages (freed when PV is done)
constexpr int kHalfBytes = kPrefillTileM * 128;          // 128 rows x 64 bf16 (one swizzle column)
constexpr int kTileBytes = 2 * kHalfBytes;               // 128 x 128 bf16
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;
constexpr int kOffV = kOffK + kNK * kTileBytes;
constexpr int kOffBar = kOffV + kNV * kTileBytes;
// barriers: q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], p_full[2],
// pv_done[2], mma_done
constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 2 + 2 + 2 + 1;
constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr int kOffFlag = kOffTmemSlot + 16;
constexpr int kSmemBytes = kOffFlag + 16;
constexpr int kSmemAlloc = kSmemBytes + 1008;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr float kRescaleSlack = 8.f;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);   // Q, K both K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);    // P from TMEM, V MN-major

struct Bars {
    uint64_t* q_full;
    uint64_t* k_full;
    uint64_t* k_empty;
    uint64_t* v_full;
    uint64_t* v_empty;
    uint64_t* s_full;
    uint64_t* p_full;
    uint64_t* pv_done;
    uint64_t* mma_done;
};

__device__ __forceinline__ Bars bars_at(uint8_t* sm) {
    uint64_t* b = reinterpret_cast<uint64_t*>(sm + kOffBar);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + kNK;
    r.v_full = r.k_empty + kNK;
    r.v_empty = r.v_full + kNV;
    r.s_full = r.v_empty + kNV;
    r.p_full = r.s_full + 2;
    r.pv_done = r.p_full + 2;
    r.mma_done = r.pv_done + 2;
    return r;
}

// Physical cache rows of the 8 pages of KV tile j (row -16 reads as zeros: past the end of
// the sequence, or a block-table entry out of range, which is also flagged).
__device__ __forceinline__ void tile_rows(const PrefillParams& p, const int32_t* btrow, int seq_pages, int kvh,
                                          int j, int rows[8]) {
#pragma unroll
    for (int pg = 0; pg < 8; ++pg) {
        const int lp = j * 8 + pg;
        int ph = -1;
        if (lp < seq_pages) {
            ph = btrow[lp];
            if (ph < 0 || ph >= p.num_pages) {
                atomicOr(p.err, PKVA_DEVERR_BAD_PAGE);
                ph = -1;
            }
        }
        rows[pg] = ph >= 0 ? (ph * p.Hkv + kvh) * kPageSize : -kPageSize;
    }
}

__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const int rows[8]) {
    mbar_arrive_expect_tx(bar, kTileBytes);
#pragma unroll
    for (int pg = 0; pg < 8; ++pg)
#pragma unroll
        for (int h = 0; h < 2; ++h) tma_load_2d(dst + h * kHalfBytes + pg * (kPageSize * 128), map, bar, h * 64, rows[pg]);
}

// Bounded wait that also gives up at once when another role already gave up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (!mbar_wait_bounded(bar, parity, err, PKVA_DEVERR_TIMEOUT)) {
        *abort_flag = 1;
        return false;
    }
    return true;
}

__global__ void __launch_bounds__(kPThreads, 1)
prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const PrefillWork w = p.work[blockIdx.x];
    const SeqInfo si = p.seqs[w.seq];
    const Bars B = bars_at(sm);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffTmemSlot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffFlag);
    const int n = w.num_kv_tiles;
    const int kvh = w.q_head / p.G;
    const int prefix = si.seq_len - si.query_len;

    if (tid == 0) {
        mbar_init(B.q_full, 1);
        for (int s = 0; s < kNK; ++s) {
            mbar_init(&B.k_full[s], 1);
            mbar_init(&B.k_empty[s], 1);
        }
        for (int s = 0; s < kNV; ++s) {
            mbar_init(&B.v_full[s], 1);
            mbar_init(&B.v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&B.s_full[b], 1);
            mbar_init(&B.p_full[b], 128);
            mbar_init(&B.pv_done[b], 1);
        }
        mbar_init(B.mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4 || warp == 6) {
        // ------------------ TMA producers: warp 4 loads Q and K, warp 6 loads V -------------
        if (lane == 0) {
            const bool is_k = warp == 4;
            const int seq_pages = (si.seq_len + kPageSize - 1) / kPageSize;
            const int32_t* btrow = p.block_table + (int64_t)w.seq * p.bt_stride;
            if (is_k) {
                prefetch_tensormap(&tmQ);
                prefetch_tensormap(&tmK);
                const int qrow0 = si.q_start + w.tok0;
                mbar_arrive_expect_tx(B.q_full, kTileBytes);
                tma_load_3d(sm + kOffQ, &tmQ, B.q_full, 0, w.q_head, qrow0);
                tma_load_3d(sm + kOffQ + kHalfBytes, &tmQ, B.q_full, 64, w.q_head, qrow0);
            } else {
                prefetch_tensormap(&tmV);
            }
            const int NSt = is_k ? kNK : kNV;
            uint64_t* full = is_k ? B.k_full : B.v_full;
            uint64_t* empty = is_k ? B.k_empty : B.v_empty;
            uint8_t* base = sm + (is_k ? kOffK : kOffV);
            for (int j = 0; j < n; ++j) {
                const int st = j % NSt;
                if (j >= NSt && !wait_or_abort(&empty[st], ((j / NSt) - 1) & 1, p.err, abort_flag)) break;
                int rows[8];
                tile_rows(p, btrow, seq_pages, kvh, j, rows);
                load_tile(base + st * kTileBytes, is_k ? &tmK : &tmV, &full[st], rows);
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer -------------------------------------------
        if (lane == 0) {
            const uint32_t q_base = smem_addr(sm + kOffQ);
            const uint32_t k_base = smem_addr(sm + kOffK);
            const uint32_t v_base = smem_addr(sm + kOffV);
            auto issue_qk = [&](int j) {
                const int st = j % kNK;
                const uint32_t d = tmem + kColS + (j & 1) * 128;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalfBytes + (ks & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(q_base + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(k_base + st * kTileBytes + off, 16, 1024);
                    tc_mma_ss(d, ad, bd, kIdescQK, ks > 0);
                }
                tc_commit(&B.s_full[j & 1]);
                tc_commit(&B.k_empty[st]);
            };
            bool ok = wait_or_abort(B.q_full, 0, p.err, abort_flag) &&
                      wait_or_abort(&B.k_full[0], 0, p.err, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_qk(0);
            }
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n) {
                    const int kst = (j + 1) % kNK;
                    if (!wait_or_abort(&B.k_full[kst], ((j + 1) / kNK) & 1, p.err, abort_flag)) break;
                    tc_fence_after();
                    issue_qk(j + 1);
                }
                const int st = j % kNV;
                if (!wait_or_abort(&B.p_full[j & 1], (j >> 1) & 1, p.err, abort_flag)) break;
                if (!wait_or_abort(&B.v_full[st], (j / kNV) & 1, p.err, abort_flag)) break;
                tc_fence_after();
                const uint32_t pcol = tmem + kColP + (j & 1) * 64;
#pragma unroll
                for (int ks = 0; ks < kPrefillTileN / 16; ++ks) {
                    const uint64_t bd = smem_desc_sw128(v_base + st * kTileBytes + ks * 2048, kHalfBytes, 1024);
                    tc_mma_ts(tmem + kColO, pcol + ks * 8, bd, kIdescPV, (j > 0 || ks > 0) ? 1u : 0u);
                }
                tc_commit(&B.pv_done[j & 1]);
                tc_commit(&B.v_empty[st]);
            }
            // every MMA this thread issued must finish before TMEM is released
            tc_commit(B.mma_done);
            mbar_wait_bounded(B.mma_done, 0, p.err, PKVA_DEVERR_TIMEOUT);
        }
    } else {
        // ------------------------------ softmax (rows) ---------------------------------------
        const int r = tid;                                   // row = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int tok = w.tok0 + r;
        const bool real_row = r < w.ntok;
        const int lim = real_row ? prefix + tok : 0x7fffffff;   // last visible key of this row
        const int lim0 = prefix + w.tok0;                        // row 0's limit
        float m_ref = -INFINITY, l_sum = 0.f;
        bool alive = true;
        // every break below is taken by the whole warp (tcgen05.ld/st are warp-collective)
        for (int j = 0; j < n; ++j) {
            if (!__all_sync(0xffffffffu, wait_or_abort(&B.s_full[j & 1], (j >> 1) & 1, p.err, abort_flag))) {
                alive = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[128];
            {
                const uint32_t sa = tmem + lane_off + kColS + (j & 1) * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(sa + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                tmem_wait_ld();
            }
            float s[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
            const int kb = j * kPrefillTileN;
            if (kb + kPrefillTileN - 1 > lim0) {            // tile crosses the diagonal
                const int vis = lim - kb;                      // columns <= vis are visible
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > vis) s[c] = -INFINITY;
            }
            // row max as eight independent chains (short dependency depth)
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
            for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
#pragma unroll
            for (int i = 0; i < 4; ++i) mx8[i] = fmaxf(mx8[i], mx8[i + 4]);
            const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3]));
            const float m_tile = mx * p.scale_log2;
            bool need = false;
            float m_new = m_ref;
            if (j == 0) {
                m_ref = m_tile;
            } else {
                need = m_tile > m_ref + kRescaleSlack;
                m_new = fmaxf(m_ref, m_tile);
            }
            if (__any_sync(0xffffffffu, need)) {
                // rescale this warp's rows of O (needs PV of tile j-1 to have landed)
                if (!__all_sync(0xffffffffu,
                                wait_or_abort(&B.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err, abort_flag))) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                const float alpha = need ? exp2f(m_ref - m_new) : 1.f;
                if (need) {
                    m_ref = m_new;
                    l_sum *= alpha;
                }
                const uint32_t oa = tmem + lane_off + kColO;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(oa + c * 32, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    tmem_st32(oa + c * 32, ov);
                }
            }
            const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
            uint32_t pk[64];
            float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = exp2f(fmaf(s[2 * c], p.scale_log2, -ref));
                const float p1 = exp2f(fmaf(s[2 * c + 1], p.scale_log2, -ref));
                ls4[c & 3] += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            l_sum += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
            // P buffer (j & 1) was last read by PV of tile j-2
            if (j >= 2 &&
                !__all_sync(0xffffffffu, wait_or_abort(&B.pv_done[j & 1], ((j - 2) >> 1) & 1, p.err, abort_flag))) {
                alive = false;
                break;
            }
            const uint32_t pa = tmem + lane_off + kColP + (j & 1) * 64;
            tmem_st32(pa, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st32(pa + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&B.p_full[j & 1]);
        }
        // ---- epilogue: O / l -> bf16 rows --------------------------------------------------
        if (alive && __all_sync(0xffffffffu, wait_or_abort(&B.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, p.err,
                                                          abort_flag))) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const uint32_t oa = tmem + lane_off + kColO;
            __nv_bfloat16* dst = p.out + ((int64_t)(si.q_start + tok) * p.Hq + w.q_head) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                tmem_ld32(oa + c * 32, ov);
                tmem_wait_ld();
                if (real_row) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
                        *reinterpret_cast<uint4*>(dst + c * 32 + e) = v;
                    }
                }
            }
        }
    }
    // all roles done (the MMA thread waited for its last MMA); release TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int prefill_ctas_per_sm() {
    int n = 0;
    if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prefill_kernel, kPThreads, kSmemAlloc) != cudaSuccess)
        return 0;
    return n;
}

cudaError_t launch_prefill(const PrefillParams& p, int num_work, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, cudaStream_t stream) {
    if (num_work == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    prefill_kernel<<<num_work, kPThreads, kSmemAlloc, stream>>>(p, tmQ, tmK, tmV);
    return cudaGetLastError();
}

}  // namespace pkva
