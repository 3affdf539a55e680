// Decode / verify attention over the paged KV cache (K-D).
//
// One CTA runs one tile task: up to 16 packed rows (token x query head of one GQA group)
// of one sequence against a range of its KV pages for one KV head. Every K and V page
// block is loaded once per task by TMA (128-byte swizzle, so the lane patterns below read
// shared memory without bank conflicts) and reused by all rows of the group: the whole
// query-head group shares one read of the page. Each of the four warps streams every
// fourth page through its own ring of stages and keeps its own online-softmax state; the
// warps merge their states at the end, and a task that is one split of a long context
// writes a partial that the last split to finish merges (flash-decoding combine).
//
// Two page bodies share that frame:
//   * decode_mma_kernel (default): the page's 16 keys are the M side of warp-level
//     tensor-core tiles (mma.sync m16n8k16, bf16 in, fp32 accumulate) and the group's
//     rows the N side: S^T = K Q^T, then O^T += V^T P^T after a transpose of P in
//     registers. About 90 instructions per page per warp, so the task stays bound by HBM
//     even for 16-row groups and draft trees.
//   * decode_fma_kernel: the same math on CUDA cores (fp32 FMA), each lane summing half a
//     head dimension for one key. It is issue-bound above 4 rows per task (measured:
//     ~830 instructions per page per warp) and is kept as the comparison point.
// Both use a warp-shuffle online softmax (running max and sum per row).
//
// Sources: XY-Serve (arXiv 2412.18106), verdict page — core_discovery (decode and verify
// tokens read a paged block cache; FlashAttention-style tiling) and forward_implications[2]
// (the visible keys are chosen per row: a causal limit for prefill/decode rows, ancestors
// in the draft tree for verify rows); supporting citation [1] (FlashAttention's QK /
// softmax / SV pattern, here with a running max and sum per row).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>


#include "pkva_decode_body.cuh"

namespace pkva {

namespace {

// Stand-alone decode kernels: four page-streaming warps per CTA (128 threads).
constexpr int kDecThreads = 128;
template <int D, int NR>
struct StandaloneNS {
    static constexpr int value = (D == 64) ? 4 : (NR <= 8 ? 3 : 2);
};

template <int D, int NT>
__global__ void __launch_bounds__(kDecThreads)
decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const dec::Group grp{(int)threadIdx.x, kDecThreads, 0};
    dec::decode_mma_task<D, NT, 4, StandaloneNS<D, NT * 8>::value>(grp, p, blockIdx.x, tmK, tmV, sm);
}

template <int D, int NR>
__global__ void __launch_bounds__(kDecThreads)
decode_fma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const dec::Group grp{(int)threadIdx.x, kDecThreads, 0};
    dec::decode_fma_task<D, NR, 4, StandaloneNS<D, NR>::value>(grp, p, blockIdx.x, tmK, tmV, sm);
}

// ---- launch plumbing ---------------------------------------------------------------------

template <class K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <class K>
int resident(K kernel, int bytes) {
    int n = 0;
    if (set_smem(kernel, bytes) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kDecThreads, bytes) != cudaSuccess) return 0;
    return n;
}

template <int D, int NR>
cudaError_t launch_t(const DecodeParams& p, int num_work, bool mma, const CUtensorMap& tmK,
                     const CUtensorMap& tmV, cudaStream_t stream) {
    if (mma) {
        constexpr int NT = NR <= 8 ? 1 : 2;
        using C = dec::DecodeCfg<D, NT * 8, false, 4, StandaloneNS<D, NT * 8>::value>;
        cudaError_t e = set_smem(decode_mma_kernel<D, NT>, C::ALLOC);
        if (e != cudaSuccess) return e;
        decode_mma_kernel<D, NT><<<num_work, kDecThreads, C::ALLOC, stream>>>(p, tmK, tmV);
    } else {
        using C = dec::DecodeCfg<D, NR, true, 4, StandaloneNS<D, NR>::value>;
        cudaError_t e = set_smem(decode_fma_kernel<D, NR>, C::ALLOC);
        if (e != cudaSuccess) return e;
        decode_fma_kernel<D, NR><<<num_work, kDecThreads, C::ALLOC, stream>>>(p, tmK, tmV);
    }
    return cudaGetLastError();
}

template <int D, int NR>
int ctas_t(bool mma) {
    if (mma) {
        constexpr int NT = NR <= 8 ? 1 : 2;
        return resident(decode_mma_kernel<D, NT>, dec::DecodeCfg<D, NT * 8, false, 4, StandaloneNS<D, NT * 8>::value>::ALLOC);
    }
    return resident(decode_fma_kernel<D, NR>, dec::DecodeCfg<D, NR, true, 4, StandaloneNS<D, NR>::value>::ALLOC);
}

}  // namespace

int decode_ctas_per_sm(int D, int rows, bool mma) {
    if (D == 64) return rows <= 4 ? ctas_t<64, 4>(mma) : rows <= 8 ? ctas_t<64, 8>(mma) : ctas_t<64, 16>(mma);
    if (D == 128) return rows <= 4 ? ctas_t<128, 4>(mma) : rows <= 8 ? ctas_t<128, 8>(mma) : ctas_t<128, 16>(mma);
    return 0;
}

cudaError_t launch_decode(const DecodeParams& p, int num_work, int D, int rows, bool mma, const CUtensorMap& tmK,
                          const CUtensorMap& tmV, cudaStream_t stream) {
    if (num_work == 0) return cudaSuccess;
    if (D == 64) {
        if (rows <= 4) return launch_t<64, 4>(p, num_work, mma, tmK, tmV, stream);
        if (rows <= 8) return launch_t<64, 8>(p, num_work, mma, tmK, tmV, stream);
        return launch_t<64, 16>(p, num_work, mma, tmK, tmV, stream);
    }
    if (rows <= 4) return launch_t<128, 4>(p, num_work, mma, tmK, tmV, stream);
    if (rows <= 8) return launch_t<128, 8>(p, num_work, mma, tmK, tmV, stream);
    return launch_t<128, 16>(p, num_work, mma, tmK, tmV, stream);
}

}  // namespace pkva
