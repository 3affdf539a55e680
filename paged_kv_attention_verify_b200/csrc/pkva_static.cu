// attn_run_static: plan-and-run in one call that allocates no device memory.
//
// Some callers cannot call cudaMalloc at the point where they need attention — for
// example an engine that hands out all device memory from its own pool up front, or code
// that must not allocate while other work owns the allocator. This entry point serves
// them: it plans the batch on the host and keeps everything the decode/verify kernel
// needs beyond its inputs and outputs (the task tables, the split-KV partials and
// counters, the device error word) in one fixed-size array in this file, reserved when
// the library is loaded. It calls no cudaMalloc, cudaFree or other allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <string>

#include "pkva.h"
#include "pkva_internal.h"
#include "pkva_kernels.h"

namespace pkva {

void set_last_error(const std::string& msg);

namespace {

// Capacity of the static scratch (the limits attn_run_static enforces).
constexpr int kStMaxSeqs = 4096;
constexpr int kStMaxTasks = 16384;
constexpr int kStMaxUnits = 4096;
constexpr int kStMaxTreeTokens = 16384;
constexpr size_t kStPartialBytes = size_t(8) << 20;   // split partial outputs (fp32)

constexpr size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
constexpr size_t kOffSeqs = 0;
constexpr size_t kOffWork = al256(kOffSeqs + kStMaxSeqs * sizeof(SeqInfo));
constexpr size_t kOffUnits = al256(kOffWork + kStMaxTasks * sizeof(DecodeWork));
constexpr size_t kOffAnc = al256(kOffUnits + kStMaxUnits * sizeof(SplitUnit));
constexpr size_t kOffCounters = al256(kOffAnc + kStMaxTreeTokens * sizeof(uint64_t));
constexpr size_t kOffErr = al256(kOffCounters + kStMaxUnits * sizeof(int32_t));
constexpr size_t kOffPartO = al256(kOffErr + sizeof(int32_t));
constexpr size_t kOffPartML = al256(kOffPartO + kStPartialBytes);
// (max, sum) pairs: one per partial row; sized for the smallest head_dim (64)
constexpr size_t kStMaxPartialRows = kStPartialBytes / (64 * sizeof(float));
constexpr size_t kStaticBytes = al256(kOffPartML + kStMaxPartialRows * 2 * sizeof(float));

}  // namespace
}  // namespace pkva

// The scratch itself: every GPU that loads this library holds it until the process exits.
static __device__ __align__(256) unsigned char g_pkva_static_scratch[pkva::kStaticBytes];

namespace pkva {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_dev_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device. In host code the array's name is
// only a stand-in, so the address comes from cudaGetSymbolAddress, once per device.
int static_scratch(unsigned char** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_last_error("attn_run_static: cannot determine the current device");
        return PKVA_ECUDA;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_pkva_static_scratch);
        if (e != cudaSuccess || !p) {
            set_last_error(std::string("attn_run_static: cudaGetSymbolAddress failed: ") + cudaGetErrorString(e));
            return PKVA_ECUDA;
        }
        g_dev_ptr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_dev_ptr[dev];
    return PKVA_OK;
}

bool encode_map(CUtensorMap* map, const void* base, int num_pages, int Hkv, int D) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_pages * Hkv * kPageSize};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kPageSize};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int too_big(const char* what, long have, long limit) {
    char buf[200];
    snprintf(buf, sizeof buf, "attn_run_static: batch needs %ld %s; the static scratch holds at most %ld",
             have, what, limit);
    set_last_error(buf);
    return PKVA_EUNSUPPORTED;
}

template <class T>
cudaError_t copy_table(unsigned char* base, size_t off, const std::vector<T>& v, cudaStream_t st) {
    if (v.empty()) return cudaSuccess;
    return cudaMemcpyAsync(base + off, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice, st);
}

}  // namespace
}  // namespace pkva

using namespace pkva;

extern "C" int attn_run_static(int num_seqs, const int32_t* seq_lens, const int32_t* query_lens,
                               const int32_t* block_table, int bt_stride, int num_pages, const int32_t* mask_kind,
                               const int32_t* parents, int num_q_heads, int num_kv_heads, int head_dim,
                               int page_size, float sm_scale, const void* q, const void* k_cache,
                               const void* v_cache, void* out, void* stream) {
    if (num_seqs == 0) return PKVA_OK;
    if (!block_table || !q || !k_cache || !v_cache || !out) {
        set_last_error("attn_run_static: NULL pointer argument");
        return PKVA_EINVAL;
    }
    for (const void* p : {(const void*)q, k_cache, v_cache, (const void*)out})
        if (reinterpret_cast<uintptr_t>(p) & 15u) {
            set_last_error("attn_run_static: tensor pointers must be 16-byte aligned");
            return PKVA_EINVAL;
        }
    // validate with the host planner before touching the device
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents, num_q_heads,
               num_kv_heads, head_dim, page_size, sm_scale, 1, 1};
    a.use_prefill_kernel = false;          // everything on the decode kernel (no TMEM, no extra tables)
    a.wide_tasks = false;                  // tasks of at most 16 rows (the stand-alone decode kernel)
    a.self_cascade = false;                // no tensor-core tasks
    HostPlan hp;
    std::string err;
    int rc = build_host_plan(a, &hp, &err);
    if (rc != PKVA_OK) {
        set_last_error("attn_run_static: " + err);
        return rc;
    }
    int dev = 0, major = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        set_last_error("attn_run_static: cannot query the current device");
        return PKVA_ECUDA;
    }
    if (major != 10) {
        set_last_error("attn_run_static: this library is built for sm_100a (B200); the current device is not");
        return PKVA_EUNSUPPORTED;
    }
    // the kernel runs on the current device and reaches that device's scratch: every
    // tensor must live there (a pointer to another GPU or to host memory is rejected)
    {
        const void* ptrs[5] = {block_table, q, k_cache, v_cache, out};
        const char* names[5] = {"block_table", "q", "k_cache", "v_cache", "out"};
        for (int i = 0; i < 5; ++i) {
            cudaPointerAttributes at{};
            if (cudaPointerGetAttributes(&at, ptrs[i]) != cudaSuccess) {
                cudaGetLastError();
                set_last_error(std::string("attn_run_static: cannot query the memory of ") + names[i]);
                return PKVA_EINVAL;
            }
            if ((at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) || at.device != dev) {
                set_last_error(std::string("attn_run_static: ") + names[i] +
                               " is not device memory of the current device");
                return PKVA_EINVAL;
            }
        }
    }
    a.num_sms = sms;
    const bool mma = decode_body_is_mma();
    a.ctas_per_sm = decode_ctas_per_sm(head_dim, hp.decode_rows, mma);
    if (a.ctas_per_sm < 1) {
        set_last_error("attn_run_static: decode kernel cannot be resident");
        return PKVA_ECUDA;
    }
    // capacity checks: reject what the fixed scratch cannot hold. Splitting long contexts
    // is the planner's choice, so first plan for fewer CTA slots (coarser splits) until
    // the split partials fit.
    const long max_slots = (long)(kStPartialBytes / ((size_t)kDecodeRowsMax * head_dim * sizeof(float)));
    while (true) {
        rc = build_host_plan(a, &hp, &err);
        if (rc != PKVA_OK) {
            set_last_error("attn_run_static: " + err);
            return rc;
        }
        if ((long)hp.num_slots <= max_slots || a.num_sms == 1) break;
        a.num_sms = (a.num_sms + 1) / 2;
    }
    if ((long)hp.seqs.size() > kStMaxSeqs) return too_big("sequences", (long)hp.seqs.size(), kStMaxSeqs);
    if ((long)hp.dwork.size() > kStMaxTasks) return too_big("tile tasks", (long)hp.dwork.size(), kStMaxTasks);
    if ((long)hp.units.size() > kStMaxUnits) return too_big("split units", (long)hp.units.size(), kStMaxUnits);
    if ((long)hp.anc.size() > kStMaxTreeTokens)
        return too_big("draft-tree tokens", (long)hp.anc.size(), kStMaxTreeTokens);
    if ((long)hp.num_slots > max_slots) return too_big("split partials", (long)hp.num_slots, max_slots);

    unsigned char* base = nullptr;
    rc = static_scratch(&base);
    if (rc != PKVA_OK) return rc;

    CUtensorMap tmK, tmV;
    if (!encode_map(&tmK, k_cache, hp.num_pages, hp.Hkv, hp.D) ||
        !encode_map(&tmV, v_cache, hp.num_pages, hp.Hkv, hp.D)) {
        set_last_error("attn_run_static: cuTensorMapEncodeTiled failed");
        return PKVA_ECUDA;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    // the array keeps the previous call's contents: counters and the error word must start
    // at zero; the tables and partials are fully written before they are read
    if (e == cudaSuccess) e = cudaMemsetAsync(base + kOffCounters, 0, kOffPartO - kOffCounters, st);
    if (e == cudaSuccess) e = copy_table(base, kOffSeqs, hp.seqs, st);
    if (e == cudaSuccess) e = copy_table(base, kOffWork, hp.dwork, st);
    if (e == cudaSuccess) e = copy_table(base, kOffUnits, hp.units, st);
    if (e == cudaSuccess) e = copy_table(base, kOffAnc, hp.anc, st);
    if (e != cudaSuccess) {
        set_last_error(std::string("attn_run_static: staging the task tables: ") + cudaGetErrorString(e));
        return PKVA_ECUDA;
    }
    DecodeParams dp;
    dp.q = static_cast<const __nv_bfloat16*>(q);
    dp.out = static_cast<__nv_bfloat16*>(out);
    dp.block_table = block_table;
    dp.seqs = reinterpret_cast<const SeqInfo*>(base + kOffSeqs);
    dp.work = reinterpret_cast<const DecodeWork*>(base + kOffWork);
    dp.units = reinterpret_cast<const SplitUnit*>(base + kOffUnits);
    dp.anc = reinterpret_cast<const uint64_t*>(base + kOffAnc);
    dp.part_o = reinterpret_cast<float*>(base + kOffPartO);
    dp.part_ml = reinterpret_cast<float*>(base + kOffPartML);
    dp.counters = reinterpret_cast<int32_t*>(base + kOffCounters);
    dp.err = reinterpret_cast<int32_t*>(base + kOffErr);
    dp.bt_stride = hp.bt_stride;
    dp.Hq = hp.Hq;
    dp.Hkv = hp.Hkv;
    dp.G = hp.G;
    dp.num_pages = hp.num_pages;
    dp.scale_log2 = hp.scale * 1.4426950408889634f;
    e = launch_decode(dp, (int)hp.dwork.size(), hp.D, hp.decode_rows, mma, tmK, tmV, st);
    if (e != cudaSuccess) {
        set_last_error(std::string("attn_run_static: launch: ") + cudaGetErrorString(e));
        return PKVA_ECUDA;
    }
    return PKVA_OK;
}
