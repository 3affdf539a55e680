// Prefill task body: causal chunked-prefill attention over the paged KV cache on 5th-generation tensor cores
// (K-P): S = Q K^T and O += P V are tcgen05.mma BF16 tiles with fp32 accumulators in
// tensor memory (TMEM).
//
// One CTA runs one task: two 128-token query tiles (tcgen05 M = 128) of query heads that
// share one KV head (two heads on the same tokens, or one head's two consecutive token
// tiles), sharing every 128-key KV tile (8 pages, gathered by TMA through the block
// table). KV tiles past a tile's last row are never loaded (causal tile skipping) and only
// tiles that cross the diagonal are masked element by element.
//
// Warp roles (352 threads):
//   warps 0-3, 4-7  two softmax warpgroups, one per query tile: thread r owns row r =
//              TMEM lane r. Each reads S, keeps the running max / sum, writes P (bf16) over
//              the first half of S in TMEM, rescales O in TMEM only when a row max moved by
//              more than 2^8, and finally writes its O rows.
//   warp 8     TMA producer of Q and of K tiles (2-stage ring, freed after both QK^T).
//   warp 9     MMA issuer (one thread) and TMEM owner. The two tiles ping-pong: while one
//              warpgroup runs its softmax, the tensor cores run the other tile's PV and
//              next QK^T. PV takes P straight from TMEM as its A operand.
//   warp 10    TMA producer of V tiles (2-stage ring, freed after both PV).
//   warp 11    (fused KV append only) copies a share of the new rows into the cache.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512); P_b lives in
// columns [0,64) of S_b (bf16 pairs). Tensor-core operations of one issuing thread run in
// issue order, so the next QK^T into S_b is issued right after the PV that reads P_b.
//
// The same body runs shared-prefix (cascade) tasks and tensor-core verify tasks: the packed
// (token, head) rows of one KV head in a query tile, the KV tiles of a shared prefix or of
// the sequence's own keys (tree / causal masks on the tiles that hold the new tokens' keys,
// which fused append patches in from the dense input). With one query tile the two
// warpgroups take alternate KV tiles and combine their halves at the end.
//
// Sources: XY-Serve (arXiv 2412.18106), verdict page — key_machinery (the attention
// primitive is a matmul-softmax-matmul tile whose QK and SV products overlap the softmax),
// core_discovery (chunked prefill on cached prefixes; fully masked tiles are skipped);
// supporting citation [1] (FlashAttention's tiled online softmax).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkva.h"
#include "pkva_append.cuh"
#include "pkva_kernels.h"
#include "pkva_merge.cuh"
#include "pkva_ptx.cuh"

namespace pkva {
namespace pre {


constexpr int kPThreads = 352;
constexpr int kPThreadsAppend = 384;                     // with the cache-writing warp
constexpr int kD = 128;
constexpr int kNK = 2;                                   // K stages
constexpr int kNV = 2;                                   // V stages
constexpr int kHalfBytes = kPrefillTileM * 128;          // 128 rows x 64 bf16 (one swizzle column)
constexpr int kTileBytes = 2 * kHalfBytes;               // 128 x 128 bf16
constexpr int kOffQ = 0;                                 // Q0, Q1
constexpr int kOffK = kOffQ + 2 * kTileBytes;
constexpr int kOffV = kOffK + kNK * kTileBytes;
constexpr int kOffBar = kOffV + kNV * kTileBytes;
// q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], p_full[2], o_ready[2], mma_done,
// v_fix, k_fix
constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 2 + 2 + 2 + 1 + 1 + 1;
constexpr int kOffFlag = kOffBar + kNumBars * 8;         // the task's abort flag
constexpr int kSmemBytes = kOffFlag + 16;

// The layout above for head_dim D (64 or 128): Q, K and V tiles are 128 rows of D bf16 in
// D / 64 swizzle halves; S stays 128 x 128 (keys), O is 128 x D.
template <int D>
struct Lay {
    static_assert(D == 64 || D == 128, "tensor-core tasks: head_dim 64 or 128");
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kHalves * kHalfBytes;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kNK * kTileBytes;
    static constexpr int kOffBar = kOffV + kNV * kTileBytes;
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);   // P from TMEM, V MN-major
};
static_assert(Lay<128>::kSmemBytes == kSmemBytes, "head_dim 128 layout");
constexpr int kSmemAlloc = kSmemBytes + 1008;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr float kRescaleSlack = 8.f;
constexpr int kWarpKProd = 8, kWarpMma = 9, kWarpVProd = 10;
constexpr bool kSpinOnS = false;   // softmax warps wait for S suspended (polling took issue slots from the other tile)

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
    uint64_t* o_ready;
    uint64_t* mma_done;
    uint64_t* v_fix;         // a V tile the producer patches before releasing it
    uint64_t* k_fix;         // a K tile the producer patches before releasing it
};

template <int D>
__device__ __forceinline__ Bars bars_at(uint8_t* sm) {
    uint64_t* b = reinterpret_cast<uint64_t*>(sm + Lay<D>::kOffBar);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + kNK;
    r.v_full = r.k_empty + kNK;
    r.v_empty = r.v_full + kNV;
    r.s_full = r.v_empty + kNV;
    r.p_full = r.s_full + 2;
    r.o_ready = r.p_full + 2;
    r.mma_done = r.o_ready + 2;
    r.v_fix = r.mma_done + 1;
    r.k_fix = r.v_fix + 1;
    return r;
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

// As wait_or_abort, polling without suspending (for waits on the critical path).
__device__ __forceinline__ bool spin_or_abort(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (!mbar_spin_bounded(bar, parity, err, PKVA_DEVERR_TIMEOUT)) {
        *abort_flag = 1;
        return false;
    }
    return true;
}

// Physical cache rows of the 8 pages of KV tile j (row -16 reads as zeros: a page with no
// key below key_limit, or a block-table entry out of range, which is also flagged).
__device__ __forceinline__ void tile_rows(const PrefillParams& p, const int32_t* btrow, int key_limit, int kvh,
                                          int j, int rows[8]) {
#pragma unroll
    for (int pg = 0; pg < 8; ++pg) {
        const int lp = j * 8 + pg;
        int ph = -1;
        if (lp * kPageSize < key_limit) {
            ph = btrow[lp];
            if (ph < 0 || ph >= p.num_pages) {
                atomicOr(p.err, PKVA_DEVERR_BAD_PAGE);
                ph = -1;
            }
        }
        rows[pg] = ph >= 0 ? (ph * p.Hkv + kvh) * kPageSize : -kPageSize;
    }
}

// The whole warp calls this: lane 0 posts the tile's bytes on `bar`, then lanes 0-7 each
// load one page (its D / 64 boxes). One thread issuing all of a tile's boxes streams about
// 20 GB/s; eight lanes about twice that (measured on B200).
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, const int rows[8],
                                          int lane) {
    if (lane == 0) mbar_arrive_expect_tx(bar, Lay<D>::kTileBytes);
    __syncwarp();
    int row = rows[0];
#pragma unroll
    for (int pg = 1; pg < 8; ++pg)
        if (lane == pg) row = rows[pg];
    if (lane < 8) {
#pragma unroll
        for (int h = 0; h < Lay<D>::kHalves; ++h)
            tma_load_2d(dst + h * kHalfBytes + lane * (kPageSize * 128), map, bar, h * 64, row);
    }
}

// One prefill task; every thread of the block (at least kPThreads) calls it; warps past
// the V producer only take part in the block barriers. `sm` is the block's 1024-aligned
// dynamic shared memory (kSmemBytes); `tmem` the block's 512 TMEM columns, allocated by
// the caller for the block's lifetime (a persistent block runs many tasks). The task's
// barriers are invalidated at its end, so the next task may reuse the memory.
// With p.append, KV tiles [0, nc) come from the cache (the committed prefix, keys at and past
// it masked) and tiles [nc, n) from the new tokens' K/V through tmKn / tmVn (tiles aligned
// at the chunk start), and warp 11 writes a share of the task's new rows into the cache.
//
// Task indices >= p.num_prefill are shared-prefix (cascade) tasks: the two query tiles hold
// (token, head) rows of one KV head for consecutive tokens of a group's members (tmQc), the
// KV tiles are a chunk of the shared prefix (all keys visible to every row), and each row's
// unnormalised output, max and sum go to the split slot its row-map entry names; the task
// then counts one arrival on every unit it touched and merges those it completed.
// A cascade task whose rows fit one query tile runs interleaved: both warpgroups hold the
// same rows (Q loaded once), tile b takes the KV tiles j with j % 2 == b, so the tensor
// cores run one half's PV and next QK^T while the other half's softmax runs, and the two
// halves' (max, sum, output) are combined before the partial is written.
#define PKVA_PREFILL_TASK prefill_task
#define PKVA_PREFILL_RS 0
#include "pkva_prefill_task.cuh"
#undef PKVA_PREFILL_TASK
#undef PKVA_PREFILL_RS

// The same task with the block's registers split between its warpgroups: the softmax
// warpgroups get 192 per thread, the producer / MMA / append warpgroup 120. Measured on the
// mixed batches, where decode blocks run beside the tensor-core blocks: 1-1.4 % faster
// (bf16 and FP8 unified, FP8 shared prefix); prefill-only launches keep prefill_task.
#define PKVA_PREFILL_TASK prefill_task_rs
#define PKVA_PREFILL_RS 1
#include "pkva_prefill_task.cuh"
#undef PKVA_PREFILL_TASK
#undef PKVA_PREFILL_RS

}  // namespace pre
}  // namespace pkva
