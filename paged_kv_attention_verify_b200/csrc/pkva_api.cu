// The C ABI (include/pkva.h): plan objects, device buffers, tensor maps and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "pkva.h"
#include "pkva_internal.h"
#include "pkva_kernels.h"

namespace pkva {

static thread_local std::string g_last_error;

// A named NVTX range over one host call (planning, a run), visible on a profiler timeline;
// without a profiler attached the push and pop do nothing.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

void set_last_error(const std::string& msg) { g_last_error = msg; }

static int cuda_fail(cudaError_t e, const char* what) {
    std::string m = std::string(what) + ": " + cudaGetErrorString(e);
    set_last_error(m);
    return e == cudaErrorMemoryAllocation ? PKVA_ENOMEM : PKVA_ECUDA;
}

#define PKVA_CUDA(call, what)                          \
    do {                                               \
        cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

bool decode_body_is_mma() {
    const char* v = getenv("PKVA_DECODE_BODY");
    return !(v && strcmp(v, "fma") == 0);
}

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// The cache viewed as a 2-D bf16 tensor [num_pages * Hkv * 16 rows, D columns]; one box
// is 16 rows (one page of one KV head) x 64 columns, stored with the 128-byte swizzle.
static bool encode_cache_map(CUtensorMap* map, const void* base, int num_pages, int Hkv, int D) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_pages * Hkv * kPageSize};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kPageSize};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// FP8 caches: K as a 2-D byte tensor [num_pages * Hkv * 16 rows, D] with one page block
// per box (128-byte swizzle at D = 128, 64-byte at D = 64); V, transposed per page block, as
// [num_pages * Hkv * D/8 rows, 128] with one block (D/8 rows) per box, unswizzled.
static bool encode_fp8_maps(CUtensorMap* mk, CUtensorMap* mv, const void* k, const void* vt, int num_pages, int Hkv,
                            int D) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint32_t estr[2] = {1, 1};
    {
        cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_pages * Hkv * kPageSize};
        cuuint64_t strides[1] = {(cuuint64_t)D};
        cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)kPageSize};
        if (fn(mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(k), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    // a transposed page block is D * 16 contiguous bytes: viewed as rows of 128 bytes so that
    // one box is D/8 wide rows (a 16-byte-wide box would take the copy engine 8x the rows)
    cuuint64_t dims[2] = {128, (cuuint64_t)num_pages * Hkv * (D / 8)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, (cuuint32_t)(D / 8)};
    return fn(mv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(vt), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q viewed as the 3-D bf16 tensor [sum T][Hq][D]; one box is 128 tokens x 64 columns of
// one head, stored with the 128-byte swizzle (the prefill kernel's A operand layout). The
// new tokens' K and V ([sum T][Hkv][D]) use the same view with Hkv heads. Cascade tasks
// read q in boxes of box_heads heads x box_tokens tokens (the (token, head) rows of one KV
// head's group, still 128-byte rows in the same swizzle).
static bool encode_q_map(CUtensorMap* map, const void* base, int total_q, int Hq, int D, int box_heads = 1,
                         int box_tokens = kPrefillTileM) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)total_q};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class T>
static int upload(T** dst, const std::vector<T>& src, int64_t* bytes) {
    *dst = nullptr;
    if (src.empty()) return PKVA_OK;
    PKVA_CUDA(cudaMalloc(dst, src.size() * sizeof(T)), "cudaMalloc(plan tables)");
    PKVA_CUDA(cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice), "upload plan");
    *bytes += (int64_t)(src.size() * sizeof(T));
    return PKVA_OK;
}

}  // namespace pkva

struct pkva_plan {
    pkva::HostPlan hp;
    int device = 0;
    int num_sms = 0;
    int decode_ctas = 0;
    bool decode_mma = true;
    bool kv_fp8 = false;                    // caches are FP8 E4M3 codes (attn_run_fp8)
    const int32_t* block_table = nullptr;
    pkva::SeqInfo* d_seqs = nullptr;
    pkva::DecodeWork* d_dwork = nullptr;
    pkva::PrefillWork* d_pwork = nullptr;
    int32_t* d_order = nullptr;             // unified launch order
    int32_t* d_order_tensor = nullptr;      // tensor-core tasks only (comparison mode)
    CUtensorMap tmQ;
    const void* tm_q = nullptr;
    pkva::SplitUnit* d_units = nullptr;
    uint64_t* d_anc = nullptr;
    float* d_part_o = nullptr;
    float* d_part_ml = nullptr;
    int32_t* d_counters = nullptr;
    int32_t* d_err = nullptr;
    void* d_qstage[2] = {nullptr, nullptr};     // attn_run_host: q staging, used alternately
    void* d_ostage = nullptr;
    cudaStream_t copy_in = nullptr;              // attn_run_host: the copies of q to the device
    cudaEvent_t ev_q_in[2] = {nullptr, nullptr};
    cudaEvent_t ev_q_used[2] = {nullptr, nullptr};
    int host_parity = 0;
    void* d_ostage_a[2] = {nullptr, nullptr};    // attn_run_host_async: out staging, used alternately
    cudaStream_t copy_out = nullptr;             // attn_run_host_async: the copies of out to the host
    cudaEvent_t ev_out_done[2] = {nullptr, nullptr};
    CUtensorMap tmK, tmV;
    const void* tm_k = nullptr;
    const void* tm_v = nullptr;
    CUtensorMap tmKn, tmVn;                 // the new tokens' K / V (fused append)
    const void* tm_kn = nullptr;
    const void* tm_vn = nullptr;
    CUtensorMap tmQc;                       // q in (token, head) tiles of one KV head (cascade)
    const void* tm_qc = nullptr;
    pkva::CascadeWork* d_cwork = nullptr;
    int32_t* d_crowmap = nullptr;
    int32_t* d_cunits = nullptr;
    // FP8 caches: bf16 staging pages of the tensor-core sequences, their block table and
    // source list, and the cache maps over them
    __nv_bfloat16* d_stage_k = nullptr;
    __nv_bfloat16* d_stage_v = nullptr;
    int32_t* d_stage_bt = nullptr;
    int32_t* d_stage_src = nullptr;
    CUtensorMap tmSK, tmSV;
    int64_t scratch_bytes = 0;
};

using namespace pkva;

static void free_plan(pkva_plan* p) {
    if (!p) return;
    cudaFree(p->d_seqs);
    cudaFree(p->d_dwork);
    cudaFree(p->d_pwork);
    cudaFree(p->d_order);
    cudaFree(p->d_order_tensor);
    cudaFree(p->d_units);
    cudaFree(p->d_cwork);
    cudaFree(p->d_crowmap);
    cudaFree(p->d_cunits);
    cudaFree(p->d_stage_k);
    cudaFree(p->d_stage_v);
    cudaFree(p->d_stage_bt);
    cudaFree(p->d_stage_src);
    cudaFree(p->d_anc);
    cudaFree(p->d_part_o);
    cudaFree(p->d_part_ml);
    cudaFree(p->d_counters);
    cudaFree(p->d_err);
    for (int b = 0; b < 2; ++b) {
        cudaFree(p->d_qstage[b]);
        if (p->ev_q_in[b]) cudaEventDestroy(p->ev_q_in[b]);
        if (p->ev_q_used[b]) cudaEventDestroy(p->ev_q_used[b]);
    }
    cudaFree(p->d_ostage);
    if (p->copy_in) cudaStreamDestroy(p->copy_in);
    for (int b = 0; b < 2; ++b) {
        cudaFree(p->d_ostage_a[b]);
        if (p->ev_out_done[b]) cudaEventDestroy(p->ev_out_done[b]);
    }
    if (p->copy_out) cudaStreamDestroy(p->copy_out);
    delete p;
}

extern "C" const char* attn_last_error(void) { return g_last_error.c_str(); }

static int plan_create(pkva_plan_t* out_plan, PlanArgs a, const int32_t* block_table, const char* who,
                       bool kv_fp8 = false) {
    NvtxRange range(who);
    const std::string name(who);
    if (!out_plan) {
        set_last_error(name + ": out_plan is NULL");
        return PKVA_EINVAL;
    }
    *out_plan = nullptr;
    const int num_seqs = a.num_seqs, head_dim = a.D;
    // row-split tasks run in the unified kernel only (not on the CUDA-core comparison body)
    a.wide_tasks = decode_body_is_mma();
    a.self_cascade = decode_body_is_mma();  // cascade tasks run in the unified kernel only
    if (num_seqs > 0 && !block_table) {
        set_last_error(name + ": block_table is NULL");
        return PKVA_EINVAL;
    }
    // validate on the host first (a bad batch never touches the device)
    {
        HostPlan probe;
        std::string err;
        const int rc = build_host_plan(a, &probe, &err);
        if (rc != PKVA_OK) {
            set_last_error(name + ": " + err);
            return rc;
        }
    }

    int dev = 0, major = 0, sms = 0;
    PKVA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    PKVA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "device attribute");
    PKVA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "device attribute");
    if (major != 10) {
        set_last_error(name + ": this library is built for sm_100a (B200); the current device is not");
        return PKVA_EUNSUPPORTED;
    }

    pkva_plan* p = new (std::nothrow) pkva_plan();
    if (!p) {
        set_last_error(name + ": out of host memory");
        return PKVA_ENOMEM;
    }
    p->device = dev;
    p->num_sms = sms;
    p->block_table = block_table;
    p->decode_mma = decode_body_is_mma();
    p->kv_fp8 = kv_fp8;

    // Decode tasks are balanced over slots of four page-streaming warps: the unified kernel
    // runs one block per SM holding three decode tasks, the stand-alone CUDA-core kernel its
    // own residency.
    {
        HostPlan probe;
        std::string err;
        build_host_plan(a, &probe, &err);
        const int blocks = p->decode_mma ? attn_ctas_per_sm(head_dim, probe.decode_rows)
                                         : decode_ctas_per_sm(head_dim, probe.decode_rows, false);
        if (blocks < 1) {
            free_plan(p);
            set_last_error(name + ": attention kernel cannot be resident (shared memory)");
            return PKVA_ECUDA;
        }
        p->decode_ctas = p->decode_mma ? kDecTasksPerBlock * blocks : blocks;
    }
    a.num_sms = sms;
    a.ctas_per_sm = p->decode_ctas;
    std::string err;
    int rc = build_host_plan(a, &p->hp, &err);
    if (rc != PKVA_OK) {
        free_plan(p);
        set_last_error(name + ": " + err);
        return rc;
    }
    if (kv_fp8 && !p->decode_mma) {
        free_plan(p);
        set_last_error(name + ": FP8 caches need the tensor-core decode body (PKVA_DECODE_BODY=fma)");
        return PKVA_EUNSUPPORTED;
    }
    if (!p->decode_mma && !p->hp.cwork.empty()) {
        free_plan(p);
        set_last_error(name + ": shared-prefix groups need the tensor-core decode body (PKVA_DECODE_BODY=fma)");
        return PKVA_EUNSUPPORTED;
    }

    const HostPlan& hp = p->hp;
#define PKVA_TRY(x)              \
    do {                         \
        int rc_ = (x);           \
        if (rc_ != PKVA_OK) {    \
            free_plan(p);        \
            return rc_;          \
        }                        \
    } while (0)
    PKVA_TRY(upload(&p->d_seqs, hp.seqs, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_dwork, hp.dwork, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_pwork, hp.pwork, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_order, hp.order, &p->scratch_bytes));
    {
        std::vector<int32_t> po;
        for (int32_t e : hp.order)
            if (e >= 0) po.push_back(e);
        PKVA_TRY(upload(&p->d_order_tensor, po, &p->scratch_bytes));
    }
    PKVA_TRY(upload(&p->d_units, hp.units, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_anc, hp.anc, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_cwork, hp.cwork, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_crowmap, hp.crowmap, &p->scratch_bytes));
    PKVA_TRY(upload(&p->d_cunits, hp.cunits, &p->scratch_bytes));
    auto alloc_zero = [&](void** ptr, size_t bytes, const char* what) -> int {
        if (bytes == 0) return PKVA_OK;
        cudaError_t e = cudaMalloc(ptr, bytes);
        if (e != cudaSuccess) return cuda_fail(e, what);
        e = cudaMemset(*ptr, 0, bytes);
        if (e != cudaSuccess) return cuda_fail(e, what);
        p->scratch_bytes += (int64_t)bytes;
        return PKVA_OK;
    };
    PKVA_TRY(alloc_zero((void**)&p->d_part_o, (size_t)hp.num_slots * kDecodeRowsMax * hp.D * sizeof(float),
                        "cudaMalloc(split partials)"));
    PKVA_TRY(alloc_zero((void**)&p->d_part_ml, (size_t)hp.num_slots * kDecodeRowsMax * 2 * sizeof(float),
                        "cudaMalloc(split partials)"));
    PKVA_TRY(alloc_zero((void**)&p->d_counters, hp.units.size() * sizeof(int32_t), "cudaMalloc(split counters)"));
    PKVA_TRY(alloc_zero((void**)&p->d_err, sizeof(int32_t), "cudaMalloc(error word)"));
    if (hp.num_stage_pages > 0) {
        PKVA_TRY(upload(&p->d_stage_bt, hp.stage_bt, &p->scratch_bytes));
        PKVA_TRY(upload(&p->d_stage_src, hp.stage_src, &p->scratch_bytes));
        const size_t bytes = (size_t)hp.num_stage_pages * hp.Hkv * kPageSize * hp.D * sizeof(__nv_bfloat16);
        PKVA_TRY(alloc_zero((void**)&p->d_stage_k, bytes, "cudaMalloc(FP8 staging pages)"));
        PKVA_TRY(alloc_zero((void**)&p->d_stage_v, bytes, "cudaMalloc(FP8 staging pages)"));
        if (!encode_cache_map(&p->tmSK, p->d_stage_k, hp.num_stage_pages, hp.Hkv, hp.D) ||
            !encode_cache_map(&p->tmSV, p->d_stage_v, hp.num_stage_pages, hp.Hkv, hp.D)) {
            free_plan(p);
            set_last_error(name + ": cuTensorMapEncodeTiled failed for the FP8 staging pages");
            return PKVA_ECUDA;
        }
    }
#undef PKVA_TRY
    set_last_error("");
    *out_plan = p;
    return PKVA_OK;
}

extern "C" int attn_plan(pkva_plan_t* out_plan, int num_seqs, const int32_t* seq_lens, const int32_t* query_lens,
                         const int32_t* block_table, int bt_stride, int num_pages, const int32_t* mask_kind,
                         const int32_t* parents, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                         float sm_scale) {
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents, num_q_heads,
               num_kv_heads, head_dim, page_size, sm_scale, 1, 1};
    return plan_create(out_plan, a, block_table, "attn_plan");
}

extern "C" int attn_plan_kv(pkva_plan_t* out_plan, int num_seqs, const int32_t* seq_lens, const int32_t* query_lens,
                            const int32_t* block_table, int bt_stride, int num_pages, const int32_t* mask_kind,
                            const int32_t* parents, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                            float sm_scale, int kv_dtype) {
    if (kv_dtype != PKVA_KV_BF16 && kv_dtype != PKVA_KV_FP8_E4M3) {
        set_last_error("attn_plan_kv: kv_dtype must be PKVA_KV_BF16 or PKVA_KV_FP8_E4M3");
        if (out_plan) *out_plan = nullptr;
        return PKVA_EINVAL;
    }
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents, num_q_heads,
               num_kv_heads, head_dim, page_size, sm_scale, 1, 1};
    const bool fp8 = kv_dtype == PKVA_KV_FP8_E4M3;
    a.use_prefill_kernel = true;     // FP8 caches: tensor-core tasks read bf16 staging copies of their pages
    a.kv_elem_bytes = fp8 ? 1 : 2;
    return plan_create(out_plan, a, block_table, "attn_plan_kv", fp8);
}

extern "C" int attn_plan_shared(pkva_plan_t* out_plan, int num_seqs, const int32_t* seq_lens,
                                const int32_t* query_lens, const int32_t* block_table, int bt_stride, int num_pages,
                                const int32_t* mask_kind, const int32_t* parents, int num_q_heads, int num_kv_heads,
                                int head_dim, int page_size, float sm_scale, const int32_t* prefix_group,
                                const int32_t* prefix_len, int num_groups) {
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents, num_q_heads,
               num_kv_heads, head_dim, page_size, sm_scale, 1, 1};
    a.prefix_group = prefix_group;
    a.prefix_len = prefix_len;
    a.num_groups = num_groups;
    return plan_create(out_plan, a, block_table, "attn_plan_shared");
}

extern "C" int attn_plan_shared_kv(pkva_plan_t* out_plan, int num_seqs, const int32_t* seq_lens,
                                   const int32_t* query_lens, const int32_t* block_table, int bt_stride,
                                   int num_pages, const int32_t* mask_kind, const int32_t* parents,
                                   int num_q_heads, int num_kv_heads, int head_dim, int page_size, float sm_scale,
                                   const int32_t* prefix_group, const int32_t* prefix_len, int num_groups,
                                   int kv_dtype) {
    if (kv_dtype != PKVA_KV_BF16 && kv_dtype != PKVA_KV_FP8_E4M3) {
        set_last_error("attn_plan_shared_kv: kv_dtype must be PKVA_KV_BF16 or PKVA_KV_FP8_E4M3");
        if (out_plan) *out_plan = nullptr;
        return PKVA_EINVAL;
    }
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents, num_q_heads,
               num_kv_heads, head_dim, page_size, sm_scale, 1, 1};
    a.prefix_group = prefix_group;
    a.prefix_len = prefix_len;
    a.num_groups = num_groups;
    const bool fp8 = kv_dtype == PKVA_KV_FP8_E4M3;
    a.kv_elem_bytes = fp8 ? 1 : 2;
    return plan_create(out_plan, a, block_table, "attn_plan_shared_kv", fp8);
}

extern "C" void attn_plan_destroy(pkva_plan_t plan) {
    if (!plan) return;
    const int dev = plan->device;
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != dev) cudaSetDevice(dev);
    cudaDeviceSynchronize();
    free_plan(plan);
    if (cur != dev) cudaSetDevice(cur);
}

extern "C" int attn_plan_get_info(pkva_plan_t plan, pkva_plan_info* info) {
    if (!plan || !info) {
        set_last_error("attn_plan_get_info: NULL argument");
        return PKVA_EINVAL;
    }
    const HostPlan& hp = plan->hp;
    info->num_seqs = hp.num_seqs;
    info->num_decode_items = (int32_t)hp.dwork.size();
    info->num_prefill_items = (int32_t)hp.pwork.size();
    info->num_split_units = (int32_t)hp.units.size();
    info->num_partial_slots = hp.num_slots;
    info->decode_rows = hp.decode_rows;
    info->kv_bytes = hp.kv_bytes;
    info->attn_flops = hp.attn_flops;
    info->scratch_bytes = plan->scratch_bytes;
    info->num_cascade_items = (int32_t)hp.cwork.size();
    info->reserved = 0;
    return PKVA_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int run_impl(pkva_plan_t plan, const void* q, const void* k_new, const void* v_new, const void* k_cache,
                    const void* v_cache, void* out, void* stream, const char* who, const float* k_scale = nullptr,
                    const float* v_scale = nullptr, bool fp8 = false) {
    NvtxRange range(who);
    const std::string name(who);
    if (!plan) {
        set_last_error(name + ": plan is NULL");
        return PKVA_EINVAL;
    }
    const HostPlan& hp = plan->hp;
    const bool append = k_new != nullptr || v_new != nullptr;
    if (fp8 != plan->kv_fp8) {
        set_last_error(name + (plan->kv_fp8 ? ": the plan is for FP8 caches (use attn_run_fp8)"
                                            : ": the plan is for bf16 caches (plan with attn_plan_kv for FP8)"));
        return PKVA_EINVAL;
    }
    if (hp.num_seqs == 0) return PKVA_OK;
    if (fp8 && (!k_scale || !v_scale)) {
        set_last_error(name + ": k_scale / v_scale is NULL");
        return PKVA_EINVAL;
    }
    if (!q || !k_cache || !v_cache || !out || (append && (!k_new || !v_new))) {
        set_last_error(name + ": NULL tensor pointer");
        return PKVA_EINVAL;
    }
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (append && (!aligned16(k_new) || !aligned16(v_new)))) {
        set_last_error(name + ": tensor pointers must be 16-byte aligned");
        return PKVA_EINVAL;
    }
    if (append && !plan->decode_mma) {
        set_last_error(name + ": the fused append runs on the tensor-core decode body only (PKVA_DECODE_BODY=fma)");
        return PKVA_EUNSUPPORTED;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (fp8 && (plan->tm_k != k_cache || plan->tm_v != v_cache)) {
        if (!encode_fp8_maps(&plan->tmK, &plan->tmV, k_cache, v_cache, hp.num_pages, hp.Hkv, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for the FP8 caches");
            return PKVA_ECUDA;
        }
        plan->tm_k = k_cache;
        plan->tm_v = v_cache;
    }
    if (plan->tm_k != k_cache) {
        if (!encode_cache_map(&plan->tmK, k_cache, hp.num_pages, hp.Hkv, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for k_cache");
            return PKVA_ECUDA;
        }
        plan->tm_k = k_cache;
    }
    if (plan->tm_v != v_cache) {
        if (!encode_cache_map(&plan->tmV, v_cache, hp.num_pages, hp.Hkv, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for v_cache");
            return PKVA_ECUDA;
        }
        plan->tm_v = v_cache;
    }
    const bool has_prefill = !hp.pwork.empty() || !hp.cwork.empty();
    if (!hp.cwork.empty() && plan->tm_qc != q) {
        if (!encode_q_map(&plan->tmQc, q, hp.total_q, hp.Hq, hp.D, hp.G, hp.cascade_tok)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for q (shared-prefix tiles)");
            return PKVA_ECUDA;
        }
        plan->tm_qc = q;
    }
    if (has_prefill && plan->tm_q != q) {
        if (!encode_q_map(&plan->tmQ, q, hp.total_q, hp.Hq, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for q");
            return PKVA_ECUDA;
        }
        plan->tm_q = q;
    }
    if (has_prefill && append && !fp8 && plan->tm_kn != k_new) {
        if (!encode_q_map(&plan->tmKn, k_new, hp.total_q, hp.Hkv, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for k_new");
            return PKVA_ECUDA;
        }
        plan->tm_kn = k_new;
    }
    if (has_prefill && append && !fp8 && plan->tm_vn != v_new) {
        if (!encode_q_map(&plan->tmVn, v_new, hp.total_q, hp.Hkv, hp.D)) {
            set_last_error(name + ": cuTensorMapEncodeTiled failed for v_new");
            return PKVA_ECUDA;
        }
        plan->tm_vn = v_new;
    }
    PrefillParams pp;
    pp.out = static_cast<__nv_bfloat16*>(out);
    pp.block_table = plan->block_table;
    pp.seqs = plan->d_seqs;
    pp.work = plan->d_pwork;
    pp.err = plan->d_err;
    pp.bt_stride = hp.bt_stride;
    pp.Hq = hp.Hq;
    pp.Hkv = hp.Hkv;
    pp.G = hp.G;
    pp.num_pages = hp.num_pages;
    pp.scale_log2 = hp.scale * 1.4426950408889634f;
    pp.num_prefill = (int32_t)hp.pwork.size();
    pp.cascade_tok = hp.cascade_tok;
    pp.cwork = plan->d_cwork;
    pp.crowmap = plan->d_crowmap;
    pp.cunits = plan->d_cunits;
    pp.anc = plan->d_anc;
    pp.units = plan->d_units;
    pp.part_o = plan->d_part_o;
    pp.part_ml = plan->d_part_ml;
    pp.counters = plan->d_counters;
    DecodeParams dp;
    dp.q = static_cast<const __nv_bfloat16*>(q);
    dp.out = static_cast<__nv_bfloat16*>(out);
    dp.block_table = plan->block_table;
    dp.seqs = plan->d_seqs;
    dp.work = plan->d_dwork;
    dp.units = plan->d_units;
    dp.anc = plan->d_anc;
    dp.part_o = plan->d_part_o;
    dp.part_ml = plan->d_part_ml;
    dp.counters = plan->d_counters;
    dp.err = plan->d_err;
    dp.bt_stride = hp.bt_stride;
    dp.Hq = hp.Hq;
    dp.Hkv = hp.Hkv;
    dp.G = hp.G;
    dp.num_pages = hp.num_pages;
    dp.scale_log2 = pp.scale_log2;
    dp.k_scale = k_scale;
    dp.v_scale = v_scale;
    if (append) {
        dp.append = 1;
        dp.k_new = static_cast<const __nv_bfloat16*>(k_new);
        dp.v_new = static_cast<const __nv_bfloat16*>(v_new);
        // the cache is written only at the new tokens' slots, which no task reads
        dp.k_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(k_cache));
        dp.v_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(v_cache));
        if (!fp8) {                    // (over FP8 caches the staging pass appends for the tensor-core tasks)
            pp.append = 1;
            pp.k_new = dp.k_new;
            pp.v_new = dp.v_new;
            pp.k_cache = dp.k_cache;
            pp.v_cache = dp.v_cache;
        }
    }
    cudaError_t e;
    if (fp8 && hp.num_stage_pages > 0) {
        // FP8 caches: stage the tensor-core sequences' pages as bf16, then the tasks read
        // those through the staging block table, with the caller's scales
        StageParams sp;
        sp.src = plan->d_stage_src;
        sp.n = hp.num_stage_pages;
        sp.block_table = plan->block_table;
        sp.bt_stride = hp.bt_stride;
        sp.num_pages = hp.num_pages;
        sp.Hkv = hp.Hkv;
        sp.seqs = plan->d_seqs;
        sp.k_codes = static_cast<uint8_t*>(const_cast<void*>(k_cache));
        sp.v_codes_t = static_cast<uint8_t*>(const_cast<void*>(v_cache));
        sp.stage_k = plan->d_stage_k;
        sp.stage_v = plan->d_stage_v;
        sp.err = plan->d_err;
        if (append) {
            sp.append = 1;
            sp.k_new = dp.k_new;
            sp.v_new = dp.v_new;
        }
        sp.k_scale = k_scale;
        sp.v_scale = v_scale;
        e = launch_stage_fp8(sp, st);
        if (e != cudaSuccess) return cuda_fail(e, (name + ": staging launch").c_str());
        pp.block_table = plan->d_stage_bt;
        pp.bt_stride = hp.stage_stride;
        pp.num_pages = hp.num_stage_pages;
        pp.k_scale = k_scale;
        pp.v_scale = v_scale;
    }
    AttnParams ap;
    ap.pre = pp;
    ap.dec = dp;
    const CUtensorMap& tmKn = fp8 ? plan->tmSK : append ? plan->tmKn : plan->tmQ;
    const CUtensorMap& tmVn = fp8 ? plan->tmSV : append ? plan->tmVn : plan->tmQ;
    if (plan->decode_mma) {
        // the whole batch in one launch
        ap.order = plan->d_order;
        ap.num_blocks = (int32_t)hp.order.size();
        ap.num_decode = (int32_t)hp.dwork.size();
        e = launch_attn(ap, hp.D, hp.decode_rows, has_prefill, plan->tmQ, plan->tmK, plan->tmV, tmKn, tmVn,
                        plan->tmQc, st, fp8);
    } else {
        // comparison mode: decode tasks on the CUDA-core kernel, prefill tasks after them
        e = launch_decode(dp, (int)hp.dwork.size(), hp.D, hp.decode_rows, false, plan->tmK, plan->tmV, st);
        if (e == cudaSuccess && has_prefill) {
            ap.order = plan->d_order_tensor;
            ap.num_blocks = (int32_t)(hp.pwork.size() + hp.cwork.size());
            ap.num_decode = 0;
            e = launch_attn(ap, hp.D, hp.decode_rows, has_prefill, plan->tmQ, plan->tmK, plan->tmV, tmKn, tmVn,
                            plan->tmQc, st);
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, (name + ": launch").c_str());
    return PKVA_OK;
}

extern "C" int attn_run(pkva_plan_t plan, const void* q, const void* k_cache, const void* v_cache, void* out,
                        void* stream) {
    return run_impl(plan, q, nullptr, nullptr, k_cache, v_cache, out, stream, "attn_run");
}

extern "C" int attn_run_append(pkva_plan_t plan, const void* q, const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, void* out, void* stream) {
    if (plan && plan->hp.num_seqs > 0 && (!k_new || !v_new)) {
        set_last_error("attn_run_append: k_new / v_new is NULL");
        return PKVA_EINVAL;
    }
    if (plan && plan->kv_fp8) {
        set_last_error("attn_run_append: the plan is for FP8 caches (use attn_run_fp8_append)");
        return PKVA_EINVAL;
    }
    return run_impl(plan, q, k_new, v_new, k_cache, v_cache, out, stream, "attn_run_append");
}

extern "C" int attn_run_fp8(pkva_plan_t plan, const void* q, const void* k_cache, const void* v_cache_t,
                            const float* k_scale, const float* v_scale, void* out, void* stream) {
    return run_impl(plan, q, nullptr, nullptr, k_cache, v_cache_t, out, stream, "attn_run_fp8", k_scale, v_scale,
                    true);
}

extern "C" int attn_run_fp8_append(pkva_plan_t plan, const void* q, const void* k_new, const void* v_new,
                                   void* k_cache, void* v_cache_t, const float* k_scale, const float* v_scale,
                                   void* out, void* stream) {
    if (plan && plan->hp.num_seqs > 0 && (!k_new || !v_new)) {
        set_last_error("attn_run_fp8_append: k_new / v_new is NULL");
        return PKVA_EINVAL;
    }
    return run_impl(plan, q, k_new, v_new, k_cache, v_cache_t, out, stream, "attn_run_fp8_append", k_scale, v_scale,
                    true);
}

// The host entries' staging: two q buffers (copied in on the plan's own stream), and either
// one out buffer (attn_run_host) or two (attn_run_host_async, copied out on a second stream).
static int host_staging(pkva_plan_t plan, size_t bytes, bool async, const char* who) {
    const std::string name(who);
    if (!plan->copy_in) {
        for (int b = 0; b < 2; ++b) {
            PKVA_CUDA(cudaMalloc(&plan->d_qstage[b], bytes), (name + ": cudaMalloc(q staging)").c_str());
            PKVA_CUDA(cudaEventCreateWithFlags(&plan->ev_q_in[b], cudaEventDisableTiming), "cudaEventCreate");
            PKVA_CUDA(cudaEventCreateWithFlags(&plan->ev_q_used[b], cudaEventDisableTiming), "cudaEventCreate");
        }
        PKVA_CUDA(cudaStreamCreateWithFlags(&plan->copy_in, cudaStreamNonBlocking), "cudaStreamCreate");
        plan->scratch_bytes += 2 * (int64_t)bytes;
    }
    if (!async && !plan->d_ostage) {
        PKVA_CUDA(cudaMalloc(&plan->d_ostage, bytes), (name + ": cudaMalloc(out staging)").c_str());
        plan->scratch_bytes += (int64_t)bytes;
    }
    if (async && !plan->copy_out) {
        for (int b = 0; b < 2; ++b) {
            PKVA_CUDA(cudaMalloc(&plan->d_ostage_a[b], bytes), (name + ": cudaMalloc(out staging)").c_str());
            PKVA_CUDA(cudaEventCreateWithFlags(&plan->ev_out_done[b], cudaEventDisableTiming), "cudaEventCreate");
        }
        PKVA_CUDA(cudaStreamCreateWithFlags(&plan->copy_out, cudaStreamNonBlocking), "cudaStreamCreate");
        plan->scratch_bytes += 2 * (int64_t)bytes;
    }
    return PKVA_OK;
}

static int run_host_impl(pkva_plan_t plan, const void* q_host, const void* k_cache, const void* v_cache,
                         void* out_host, void* stream, bool async, const char* who) {
    NvtxRange range(who);
    const std::string name(who);
    if (!plan) {
        set_last_error(name + ": plan is NULL");
        return PKVA_EINVAL;
    }
    const HostPlan& hp = plan->hp;
    if (hp.num_seqs == 0) return PKVA_OK;
    if (!q_host || !out_host) {
        set_last_error(name + ": NULL host pointer");
        return PKVA_EINVAL;
    }
    const size_t bytes = (size_t)hp.total_q * hp.Hq * hp.D * 2;
    const int rc0 = host_staging(plan, bytes, async, who);
    if (rc0 != PKVA_OK) return rc0;
    // q goes in on the plan's own copy stream, into the staging buffer the call before the
    // last one used, so that it overlaps the previous call's attention and copy out; the
    // attention (on `stream`) waits for it
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int b = plan->host_parity;
    plan->host_parity ^= 1;
    PKVA_CUDA(cudaStreamWaitEvent(plan->copy_in, plan->ev_q_used[b], 0), "order q staging reuse");
    PKVA_CUDA(cudaMemcpyAsync(plan->d_qstage[b], q_host, bytes, cudaMemcpyHostToDevice, plan->copy_in),
              "copy q to device");
    PKVA_CUDA(cudaEventRecord(plan->ev_q_in[b], plan->copy_in), "record q copy");
    PKVA_CUDA(cudaStreamWaitEvent(st, plan->ev_q_in[b], 0), "order attention after q copy");
    void* ostage = plan->d_ostage;
    if (async) {
        // the out buffer is free once the copy out of the call before the last one is done
        ostage = plan->d_ostage_a[b];
        PKVA_CUDA(cudaStreamWaitEvent(st, plan->ev_out_done[b], 0), "order out staging reuse");
    }
    const int rc = attn_run(plan, plan->d_qstage[b], k_cache, v_cache, ostage, stream);
    if (rc != PKVA_OK) return rc;
    PKVA_CUDA(cudaEventRecord(plan->ev_q_used[b], st), "record attention done");
    if (!async) {
        // the copy out stays on `stream`: the result is complete when `stream` reaches here
        PKVA_CUDA(cudaMemcpyAsync(out_host, ostage, bytes, cudaMemcpyDeviceToHost, st), "copy out to host");
        return PKVA_OK;
    }
    // the copy out on the plan's second stream, overlapping the next call's attention
    PKVA_CUDA(cudaStreamWaitEvent(plan->copy_out, plan->ev_q_used[b], 0), "order copy out after attention");
    PKVA_CUDA(cudaMemcpyAsync(out_host, ostage, bytes, cudaMemcpyDeviceToHost, plan->copy_out), "copy out to host");
    PKVA_CUDA(cudaEventRecord(plan->ev_out_done[b], plan->copy_out), "record copy out");
    return PKVA_OK;
}

extern "C" int attn_run_host(pkva_plan_t plan, const void* q_host, const void* k_cache, const void* v_cache,
                             void* out_host, void* stream) {
    return run_host_impl(plan, q_host, k_cache, v_cache, out_host, stream, false, "attn_run_host");
}

extern "C" int attn_run_host_async(pkva_plan_t plan, const void* q_host, const void* k_cache, const void* v_cache,
                                   void* out_host, void* stream) {
    return run_host_impl(plan, q_host, k_cache, v_cache, out_host, stream, true, "attn_run_host_async");
}

extern "C" int attn_host_wait(pkva_plan_t plan, void* stream) {
    if (!plan) {
        set_last_error("attn_host_wait: plan is NULL");
        return PKVA_EINVAL;
    }
    if (!plan->copy_out) return PKVA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int b = 0; b < 2; ++b)
        PKVA_CUDA(cudaStreamWaitEvent(st, plan->ev_out_done[b], 0), "attn_host_wait: order after copies out");
    return PKVA_OK;
}

extern "C" int attn_check(pkva_plan_t plan, void* stream, int32_t* device_error) {
    if (!plan) {
        set_last_error("attn_check: plan is NULL");
        return PKVA_EINVAL;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    PKVA_CUDA(cudaStreamSynchronize(st), "attn_check: stream synchronize");
    int32_t e = 0;
    PKVA_CUDA(cudaMemcpy(&e, plan->d_err, sizeof e, cudaMemcpyDeviceToHost), "attn_check: read error word");
    if (device_error) *device_error = e;
    if (e != 0) {
        PKVA_CUDA(cudaMemset(plan->d_err, 0, sizeof(int32_t)), "attn_check: clear error word");
        char buf[96];
        snprintf(buf, sizeof buf, "attn_check: device error bits 0x%x", (unsigned)e);
        set_last_error(buf);
        return PKVA_EDEVICE;
    }
    return PKVA_OK;
}
