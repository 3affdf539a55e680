// Launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkva_internal.h"

namespace pkva {

struct DecodeParams {
    const __nv_bfloat16* q;      // [sum T, Hq, D]
    __nv_bfloat16* out;          // [sum T, Hq, D]
    const int32_t* block_table;  // [B, bt_stride]
    const SeqInfo* seqs;
    const DecodeWork* work;
    const SplitUnit* units;
    const uint64_t* anc;         // TREE ancestor-or-self masks
    float* part_o;               // [slots, kDecodeRowsMax, D]: unnormalised split outputs
    float* part_ml;              // [slots, kDecodeRowsMax, 2]: (max, sum) in log2 units
    int32_t* counters;           // [units]: split tasks finished (reset by the last one)
    int32_t* err;                // device error word
    int32_t bt_stride;
    int32_t Hq, Hkv, G;
    int32_t num_pages;
    float scale_log2;            // softmax scale * log2(e)
    // fused KV append (attn_run_append): the new tokens' K/V, in q's token order
    int32_t append = 0;
    const __nv_bfloat16* k_new = nullptr;  // [sum T, Hkv, D]
    const __nv_bfloat16* v_new = nullptr;
    __nv_bfloat16* k_cache = nullptr;      // written at the new tokens' slots
    __nv_bfloat16* v_cache = nullptr;
    // FP8 (E4M3) caches: one float scale per KV head for K and for V
    const float* k_scale = nullptr;
    const float* v_scale = nullptr;
};

struct PrefillParams {
    __nv_bfloat16* out;          // [sum T, Hq, 128]
    const int32_t* block_table;  // [B, bt_stride]
    const SeqInfo* seqs;
    const PrefillWork* work;
    int32_t* err;
    int32_t bt_stride;
    int32_t Hq, Hkv, G;
    int32_t num_pages;
    float scale_log2;
    int32_t append = 0;          // fused KV append: see DecodeParams
    const __nv_bfloat16* k_new = nullptr;
    const __nv_bfloat16* v_new = nullptr;
    __nv_bfloat16* k_cache = nullptr;
    __nv_bfloat16* v_cache = nullptr;
    // shared-prefix (cascade) tasks: task indices >= num_prefill
    int32_t num_prefill = 0;
    int32_t cascade_tok = 0;     // tokens per 128-row tile: floor(128 / G)
    const CascadeWork* cwork = nullptr;
    const int32_t* crowmap = nullptr;    // [tasks][256]: partial index slot*16 + row, or -1
    const int32_t* cunits = nullptr;
    const uint64_t* anc = nullptr;       // tree ancestor masks (tensor-core verify tasks)
    const SplitUnit* units = nullptr;
    float* part_o = nullptr;
    float* part_ml = nullptr;
    int32_t* counters = nullptr;
    // FP8 caches: the tasks read bf16 copies of the codes (block_table / num_pages address
    // the staging pages); the K scale of the task's KV head multiplies the softmax scale and
    // the V scale the output
    const float* k_scale = nullptr;
    const float* v_scale = nullptr;
};

// FP8 caches: copy the pages of the tensor-core sequences to bf16 staging pages (the codes'
// exact values, unscaled), one block per staging page and all KV heads. Slots past the
// sequence's end become zeros. With append, the new tokens' codes are computed from
// k_new / v_new, written into the FP8 caches and staged.
struct StageParams {
    const int32_t* src;          // [n][2]: (sequence, logical page)
    int32_t n;                   // staging pages
    const int32_t* block_table;  // the caller's [B, bt_stride]
    int32_t bt_stride;
    int32_t num_pages;           // the caller's page pool
    int32_t Hkv;
    const SeqInfo* seqs;
    uint8_t* k_codes;            // [pages, Hkv, 16, 128]
    uint8_t* v_codes_t;          // [pages, Hkv, 128, 16]
    __nv_bfloat16* stage_k;      // [n, Hkv, 16, 128]
    __nv_bfloat16* stage_v;
    int32_t* err;
    int32_t append = 0;
    const __nv_bfloat16* k_new = nullptr;   // [sum T, Hkv, 128]
    const __nv_bfloat16* v_new = nullptr;
    const float* k_scale = nullptr;
    const float* v_scale = nullptr;
};
cudaError_t launch_stage_fp8(const StageParams& p, cudaStream_t stream);

// Everything one launch of the unified attention kernel needs.
// One entry of `order` per block: e >= 0 runs tensor-core task e (a prefill task, or
// cascade task e - num_prefill); e < 0 runs decode tasks 3(-1-e) .. 3(-1-e)+2 side by side.
struct AttnParams {
    PrefillParams pre;
    DecodeParams dec;
    const int32_t* order;
    int32_t num_blocks;
    int32_t num_decode;           // decode/verify tasks
};

// Resident blocks per SM of the unified kernel (one: each block takes most of an SM).
int attn_ctas_per_sm(int D, int rows);

// Launch the unified kernel over p.num_blocks blocks in the order p.order (prefill tasks
// need head_dim 128). tmQ views q as the 3-D tensor [sum T][Hq][128] with a
// {64, 1, 128} box; tmK/tmV are the cache maps (16 x 64 boxes).
// tmKn/tmVn view k_new/v_new like tmQ ({64, 1, 128} boxes); read only when p.pre.append.
// tmQc views q in boxes of {64 columns, G heads, floor(128 / G) tokens}; read only by
// cascade tasks.
// fp8: the caches are E4M3 codes (tmK over [pages*Hkv*16][D] bytes, tmV over the transposed
// [pages*Hkv*D][16] bytes, read by decode/verify tasks); tensor-core tasks then read the bf16
// staging pages through tmKn / tmVn (cache maps, 16 x 64 boxes), and p.pre.append is 0.
cudaError_t launch_attn(const AttnParams& p, int D, int rows, bool has_prefill, const CUtensorMap& tmQ,
                        const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKn,
                        const CUtensorMap& tmVn, const CUtensorMap& tmQc, cudaStream_t stream, bool fp8 = false);

// Resident CTAs per SM of the decode kernel compiled for (D, rows); 0 if unsupported.
// `mma` selects the tensor-core page body, otherwise the CUDA-core one.
int decode_ctas_per_sm(int D, int rows, bool mma);

// Launch the decode/verify kernel over `num_work` tasks.
cudaError_t launch_decode(const DecodeParams& p, int num_work, int D, int rows, bool mma,
                          const CUtensorMap& tmK, const CUtensorMap& tmV, cudaStream_t stream);

// Page body for decode/verify tasks: tensor cores unless PKVA_DECODE_BODY=fma is set in
// the environment when the plan is made (the CUDA-core body, kept for comparison).
bool decode_body_is_mma();

}  // namespace pkva
