// One launch for a whole mixed prefill / decode / verify batch.
//
// The planner's task list is one grid: shared-prefix (cascade) tasks first, then prefill
// tasks and decode/verify tasks, each heaviest first, merged in proportion. A block whose
// entry is a tensor-core task runs it with all its warps (TMEM, tcgen05.mma, four warp
// roles); any other block runs three decode/verify tasks side by side, each on four warps
// with its own third of shared memory and its own named barrier (warp-level tensor-core
// page body): a task of at most 16 packed rows streams every fourth page on each warp; a
// wider one (a draft tree times the GQA group) is row-split, three warps owning 16 rows
// each and the fourth streaming every page once. Both kinds use the same 384-thread block
// and the same dynamic shared memory (one block per SM), so the hardware block scheduler
// deals the mixed work out as one longest-task-first schedule and decode blocks fill the
// SMs as prefill blocks finish.
//
// (A persistent variant, blocks pulling tasks from two global queues with each decode
// group taking its next task on its own, measured 3-13 % slower on B200 and was dropped:
// the extra per-task fetch and the register pressure of the loop outweighed the gain.)
//
// XY-Serve (arXiv 2412.18106), verdict page — forward_implications[2] (one attention kernel
// for prefill, decode and verify rows, the visible keys chosen row by row) and
// core_discovery (a budgeted mixed batch decomposed into tile tasks, reordered for balance).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkva_decode_body.cuh"
#include "pkva_prefill_body.cuh"

namespace pkva {

namespace {

constexpr int kAttnThreads = 384;                 // prefill uses 352; decode 3 x 128
constexpr int kDecWarps = 4;                      // page-streaming warps per decode task
static_assert(kAttnThreads >= pre::kPThreadsAppend, "block too small for a prefill task");
static_assert(kAttnThreads == kDecTasksPerBlock * 128, "one 128-thread group per decode task");
// prefill_task_rs splits a block's registers as 2 x 128 threads x 192 + 128 x 120: exactly the
// 384 x 168 a block is launched with (a larger split would wait for registers forever)
constexpr int kSplitLaunchRegs = 168;
static_assert(2 * 128 * 192 + 128 * 120 == kAttnThreads * kSplitLaunchRegs, "register split");

template <int D, bool FP8 = false>
struct AttnNS {
    // decode stages per warp: 16 KB of pages in flight per warp in every form
    static constexpr int value = (D == 64 ? 4 : 2) * (FP8 ? 2 : 1);
};

// TC: the kernel can run tensor-core tasks (head_dim 128 only). Launches without any
// tensor-core task use the TC = false kernel: smaller code for the decode-only plans.
template <int D, int NT, bool FP8 = false, bool TC = true>
struct AttnSmem {
    using DC = dec::DecodeCfg<D, NT * 8, false, kDecWarps, AttnNS<D, FP8>::value, FP8 ? 1 : 2>;
    static_assert(dec::DecodeCfg<D, 8, false, kDecWarps, AttnNS<D, FP8>::value, FP8 ? 1 : 2>::BYTES <= DC::BYTES,
                  "one-n-tile tasks fit a task's share");
    static constexpr int GROUP_BYTES = (DC::BYTES + 1023) / 1024 * 1024;    // one decode task
    static constexpr int DEC_BYTES = kDecTasksPerBlock * GROUP_BYTES;
    static constexpr int TASK_BYTES =
        (TC && pre::Lay<D>::kSmemBytes > DEC_BYTES) ? pre::Lay<D>::kSmemBytes : DEC_BYTES;
    static constexpr int OFF_SCHED = TASK_BYTES;  // the TMEM address of a tensor-core block
    static constexpr int BYTES = TASK_BYTES + 64;
    static constexpr int ALLOC = BYTES + 1008;    // room to align to 1024
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    // a row-split (wide) task takes one decode task's share: as many ring stages as fit
    static constexpr int WIDE_NS = dec::wide_stages(D, GROUP_BYTES);
    static_assert(dec::wide_bytes(D, WIDE_NS) <= GROUP_BYTES, "wide task");
};

// FP8: decode/verify tasks read the E4M3 pages; tensor-core tasks read their bf16 staging copies.
// Tensor-core tasks run at head_dim 128 and, over bf16 caches, 64.
// TCM: 0 no tensor-core tasks; 1 tensor-core tasks; 2 tensor-core tasks beside decode blocks,
// run as prefill_task_rs (the block's registers split between its warpgroups)
template <int D, int NT, bool FP8, int TCM>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKn,
            const __grid_constant__ CUtensorMap tmVn, const __grid_constant__ CUtensorMap tmQc) {
    constexpr bool TC = TCM != 0;
    using S = AttnSmem<D, NT, FP8, TC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int e = p.order[blockIdx.x];
    if constexpr (TC) {
        if (e >= 0) {
            // tensor-core task: 512 TMEM columns for the block (one block per SM)
            uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::OFF_SCHED);
            const int warp = threadIdx.x >> 5;
            if (warp == pre::kWarpMma) {
                tmem_alloc(tmem_slot, pre::kTmemCols);
                tmem_relinquish();
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            const uint32_t tmem = *tmem_slot;
            // over FP8 caches the tensor-core tasks read the bf16 staging pages (tmKn / tmVn)
            if constexpr (TCM == 2)
                pre::prefill_task_rs<D>(p.pre, e, tmQ, FP8 ? tmKn : tmK, FP8 ? tmVn : tmV, tmKn, tmVn, tmQc, tmem, sm);
            else
                pre::prefill_task<D>(p.pre, e, tmQ, FP8 ? tmKn : tmK, FP8 ? tmVn : tmV, tmKn, tmVn, tmQc, tmem, sm);
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (warp == pre::kWarpMma) tmem_dealloc(tmem, pre::kTmemCols);
            return;
        }
    }
    if (e >= 0) return;                          // (never planned: a launch without tensor-core code)
    // decode block: warps 4g .. 4g+3 run task g of the block's three
    const int g = threadIdx.x >> 7;
    const int task = (-1 - e) * kDecTasksPerBlock + g;
    if (task >= p.num_decode) return;
    const dec::Group grp{(int)threadIdx.x & 127, 128, 1 + g};
    if constexpr (!FP8) {
        // more than 16 packed rows (a draft tree times the GQA group): one pass over the pages
        if (p.dec.work[task].row_count > kDecodeRowsMax) {
            dec::decode_wide_task<D, S::WIDE_NS>(grp, p.dec, task, tmK, tmV, sm + g * S::GROUP_BYTES);
            return;
        }
    }
    if constexpr (NT == 2) {
        // a launch compiled for 16-row tasks runs its tasks of at most 8 rows (decode steps
        // beside 16-row verify chunks) on the one-n-tile body
        if (p.dec.work[task].row_count <= 8) {
            dec::decode_mma_task<D, 1, kDecWarps, AttnNS<D, FP8>::value, FP8>(grp, p.dec, task, tmK, tmV,
                                                                           sm + g * S::GROUP_BYTES);
            return;
        }
    }
    dec::decode_mma_task<D, NT, kDecWarps, AttnNS<D, FP8>::value, FP8>(grp, p.dec, task, tmK, tmV,
                                                                    sm + g * S::GROUP_BYTES);
}

// The register split is used only where the compiled kernel is launched with exactly the
// registers it divides; otherwise the launch falls back to the unsplit task body.
template <int D, int NT, bool FP8>
bool split_fits() {
    static const bool ok = [] {
        cudaFuncAttributes a{};
        return cudaFuncGetAttributes(&a, attn_kernel<D, NT, FP8, 2>) == cudaSuccess && a.numRegs == kSplitLaunchRegs;
    }();
    return ok;
}

template <int D, int NT, bool FP8, int TCM>
cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                     const CUtensorMap& tmKn, const CUtensorMap& tmVn, const CUtensorMap& tmQc,
                     cudaStream_t stream) {
    if constexpr (TCM == 2)
        if (!split_fits<D, NT, FP8>()) return launch_t<D, NT, FP8, 1>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream);
    using S = AttnSmem<D, NT, FP8, TCM != 0>;
    cudaError_t e =
        cudaFuncSetAttribute(attn_kernel<D, NT, FP8, TCM>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::ALLOC);
    if (e != cudaSuccess) return e;
    const int grid = p.num_blocks;
    if (grid == 0) return cudaSuccess;
    attn_kernel<D, NT, FP8, TCM><<<grid, kAttnThreads, S::ALLOC, stream>>>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc);
    return cudaGetLastError();
}

template <int D, int NT>
int ctas_t() {
    constexpr bool TC = true;
    using S = AttnSmem<D, NT, false, TC>;
    int n = 0;
    if (cudaFuncSetAttribute(attn_kernel<D, NT, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             S::ALLOC) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, attn_kernel<D, NT, false, 1>, kAttnThreads, S::ALLOC) !=
        cudaSuccess)
        return 0;
    return n;
}

template <bool FP8, int TCM>
cudaError_t launch_kv(const AttnParams& p, int D, int rows, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                      const CUtensorMap& tmV, const CUtensorMap& tmKn, const CUtensorMap& tmVn,
                      const CUtensorMap& tmQc, cudaStream_t stream) {
    if (D == 64) {
        // head_dim 64 tensor-core tasks run over bf16 caches only (the FP8 staging copies are
        // head_dim 128)
        constexpr int TCM64 = FP8 ? 0 : TCM;
        return rows <= 8 ? launch_t<64, 1, FP8, TCM64>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
                         : launch_t<64, 2, FP8, TCM64>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream);
    }
    return rows <= 8 ? launch_t<128, 1, FP8, TCM>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
                     : launch_t<128, 2, FP8, TCM>(p, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream);
}

}  // namespace

int attn_ctas_per_sm(int D, int rows) {
    if (D == 64) return rows <= 8 ? ctas_t<64, 1>() : ctas_t<64, 2>();
    if (D == 128) return rows <= 8 ? ctas_t<128, 1>() : ctas_t<128, 2>();
    return 0;
}

cudaError_t launch_attn(const AttnParams& p, int D, int rows, bool has_prefill, const CUtensorMap& tmQ,
                        const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKn,
                        const CUtensorMap& tmVn, const CUtensorMap& tmQc, cudaStream_t stream, bool fp8) {
    if (D == 64 && fp8 && has_prefill) return cudaErrorInvalidValue;   // (never planned)
    // plans without tensor-core tasks launch the code without the prefill body; plans with
    // tensor-core and decode tasks the one whose tensor-core blocks split their registers
    const bool mixed = has_prefill && p.num_decode > 0;
    if (!fp8)
        return mixed ? launch_kv<false, 2>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
               : has_prefill ? launch_kv<false, 1>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
                             : launch_kv<false, 0>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream);
    return mixed ? launch_kv<true, 2>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
           : has_prefill ? launch_kv<true, 1>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream)
                         : launch_kv<true, 0>(p, D, rows, tmQ, tmK, tmV, tmKn, tmVn, tmQc, stream);
}

}  // namespace pkva
