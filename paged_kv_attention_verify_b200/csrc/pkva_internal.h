// Internal types shared by the host planner and the kernels (not part of the C ABI).
#pragma once

#include <stdint.h>

#include <string>
#include <vector>

namespace pkva {

constexpr int kPageSize = 16;          // keys per page (the only page size supported)
constexpr int kMaxTreeTokens = 64;     // draft tokens per TREE sequence (one 64-bit mask)
constexpr int kDecodeRowsMax = 16;     // packed (token, head) rows per decode task
constexpr int kWideRowsMax = 48;       // packed rows per row-split (wide) decode/verify task
constexpr int kDecodeMaxPages = 1024;  // pages per decode task (block-table slice in smem)
constexpr int kPrefillTileM = 128;     // query tokens per prefill tile (tcgen05 M)
constexpr int kPrefillTileN = 128;     // keys per prefill KV tile (8 pages)
constexpr int kDecTasksPerBlock = 3;   // decode tasks side by side in one block of the unified kernel
constexpr int kPrefillMinTokens = 64;  // causal sequences with at least this many new tokens
                                       // (and head_dim 128) run on the tensor-core prefill kernel
constexpr int kCascadeTilesPerTask = 16; // shared-prefix KV tiles (128 keys) per cascade task
constexpr int kOwnMinKeys = 512;         // keys from which a verify tree's rows run on the tensor cores
constexpr int kOwnTilesPerTask = 32;     // KV tiles (128 keys) per tensor-core verify task

// Per-sequence record (the "Token-Table" row of the batch).
struct SeqInfo {
    int32_t seq_len;     // L: total keys, new tokens included
    int32_t query_len;   // T: new query tokens
    int32_t q_start;     // first row of this sequence in q / out
    int32_t mask_kind;   // 0 causal, 1 tree
    int32_t anc_off;     // TREE: index of token 0's ancestor mask in the mask array
    int32_t shared_len;  // keys shared with its prefix group and read by cascade tasks (else 0)
    int32_t pad1, pad2;
};
static_assert(sizeof(SeqInfo) == 32, "SeqInfo layout");

// One decode/verify tile task (the "Task-Table" row): packed rows [row_begin,
// row_begin + row_count) of (seq, kv_head), keys of pages [page_begin, page_end).
struct DecodeWork {
    int32_t seq;
    int32_t kv_head;
    int32_t row_begin;   // packed row = token * group + head-in-group
    int32_t row_count;   // <= kDecodeRowsMax; up to kWideRowsMax for a row-split task, whose
                         // 16-row chunks are split units unit, unit + 1, ... when split
    int32_t page_begin;  // logical pages of the sequence
    int32_t page_end;
    int32_t unit;        // split unit id, -1 when the task covers its whole unit
    int32_t split;       // split index within the unit
};
static_assert(sizeof(DecodeWork) == 32, "DecodeWork layout");

// One prefill task: two tcgen05 query tiles of up to 128 tokens each, of query heads that
// share one KV head: tile 0 holds tokens [tok0, tok0 + ntok0) of q_head, tile 1 tokens
// [tok1, tok1 + ntok1) of q_head1 (ntok1 = 0: no tile 1). Usually the two tiles are two heads
// of one token tile (they need the same KV tiles); a head left over in an odd group pairs
// two consecutive token tiles of its own. Tile 0 needs KV tiles [0, kv_tiles0) of 128 keys,
// tile 1 [0, kv_tiles1).
struct PrefillWork {
    int32_t seq;
    int32_t q_head;
    int32_t tok0;
    int32_t ntok0;
    int32_t q_head1;
    int32_t tok1;
    int32_t ntok1;
    int32_t kv_tiles0;
    int32_t kv_tiles1;
    // with a fused KV append, keys come from the cache for the committed prefix (tiles
    // aligned at key 0) and from the new tokens' input for the chunk (tiles aligned at the
    // chunk start): the tile counts of the two query tiles in that mode
    int32_t kv_tiles0_append;
    int32_t kv_tiles1_append;
    int32_t pad;
};
static_assert(sizeof(PrefillWork) == 48, "PrefillWork layout");

// A (seq, kv_head, row chunk) whose keys are split over several tasks: where its partials
// live, how many task arrivals complete it, and which output rows it owns (so that any
// contributing task, decode or cascade, can merge it when it arrives last).
struct SplitUnit {
    int32_t slot_base;   // first partial slot
    int32_t num_splits;  // partial slots: decode splits, then cascade splits
    int32_t arrivals;    // tasks that must finish before the merge
    int32_t seq;
    int32_t kv_head;
    int32_t row_begin;   // packed rows [row_begin, row_begin + row_count)
    int32_t row_count;
    int32_t pad;
};
static_assert(sizeof(SplitUnit) == 32, "SplitUnit layout");

// One shared-prefix (cascade) task: the stacked query rows of a run of sequences that share
// their first prefix_len keys, against KV tiles [tile_begin, tile_end) of that prefix, as
// two tcgen05 M = 128 tiles of (token, head) rows of one KV head. Each row's partial goes to
// the split slot the row map gives; the units it touches are listed for the arrival count.
struct CascadeWork {
    int32_t lead_seq;    // the sequence whose block table supplies the shared pages
    int32_t kv_head;
    int32_t tok0;        // first q row (global token index) of the task
    int32_t ntok;        // tokens in the task (<= 2 * tokens per tile)
    int32_t tile_begin;  // KV tiles of 128 keys
    int32_t tile_end;
    int32_t unit_off;    // into the cascade unit list
    int32_t unit_cnt;
    int32_t own;         // 0: a shared prefix; 1: the rows of one sequence over a chunk of its
                         // own keys [0, seq_len) with the tree / causal masks (tensor-core
                         // verify task), partials to split slots; 2: as 1, over all of its
                         // keys, writing the output rows itself
    int32_t pad[3];
};
static_assert(sizeof(CascadeWork) == 48, "CascadeWork layout");

// Host-side result of planning, before anything is uploaded.
struct HostPlan {
    int num_seqs = 0, Hq = 0, Hkv = 0, G = 0, D = 0;
    int bt_stride = 0, num_pages = 0;
    int total_q = 0;
    float scale = 0.f;
    int decode_rows = 4;                  // rows per decode task the launch compiles for
    std::vector<SeqInfo> seqs;
    std::vector<uint64_t> anc;            // per TREE token: ancestor-or-self bit mask
    std::vector<DecodeWork> dwork;        // launch order
    std::vector<PrefillWork> pwork;       // heaviest first
    // Unified launch order, one entry per block: e >= 0 runs tensor-core task e (prefill task
    // e, or cascade task e - pwork.size()); e < 0 runs decode tasks 3*(-1-e) .. 3*(-1-e)+2
    // side by side. Cascade tasks first, then prefill and decode tasks, each heaviest
    // first, merged in proportion.
    std::vector<int32_t> order;
    std::vector<SplitUnit> units;
    int num_slots = 0;
    // shared-prefix (cascade) tasks: launch-order entries e >= pwork.size() run cascade task
    // e - pwork.size(); 2 * 128 row-map entries per task (partial index slot*16 + row, or -1)
    std::vector<CascadeWork> cwork;
    std::vector<int32_t> crowmap;
    std::vector<int32_t> cunits;
    int cascade_tok = 0;                  // tokens per cascade tile: floor(128 / G)
    // FP8 caches: the pages of the tensor-core (prefill) sequences are staged as bf16 before
    // the attention launch. Staging page n holds (sequence stage_src[2n], logical page
    // stage_src[2n+1]); stage_bt [num_seqs][stage_stride] maps a prefill sequence's logical
    // pages to staging pages (-1 elsewhere).
    std::vector<int32_t> stage_src;
    std::vector<int32_t> stage_bt;
    int stage_stride = 0;
    int num_stage_pages = 0;
    int64_t kv_bytes = 0;
    int64_t attn_flops = 0;
};

struct PlanArgs {
    int num_seqs;
    const int32_t* seq_lens;
    const int32_t* query_lens;
    int bt_stride;
    int num_pages;
    const int32_t* mask_kind;
    const int32_t* parents;
    int Hq, Hkv, D, page_size;
    float sm_scale;
    int num_sms;
    int ctas_per_sm;
    bool use_prefill_kernel = true;       // false: every sequence goes to the decode kernel
    int kv_elem_bytes = 2;                // bytes per cached K/V element (2 bf16, 1 FP8)
    // rows of a (sequence, KV head) beyond one 16-row task go to row-split tasks of up to
    // 48 rows that read each page once (the unified kernel's bf16 decode/verify path); false:
    // every task holds at most 16 rows (the stand-alone decode kernels)
    bool wide_tasks = true;
    // verify trees / short causal chunks of 17 to 128 packed rows per KV head on the
    // tensor cores (cascade-style tasks over their own keys); false: decode/verify tasks only
    bool self_cascade = true;
    // shared-prefix groups (may be NULL / 0): prefix_group[s] in {-1} U [0, num_groups),
    // members of a group consecutive in the batch, prefix_len[g] keys shared (page multiple)
    const int32_t* prefix_group = nullptr;
    const int32_t* prefix_len = nullptr;
    int num_groups = 0;
};

// Validates and decomposes; returns a pkva_status and fills `err` on failure.
int build_host_plan(const PlanArgs& a, HostPlan* out, std::string* err);

}  // namespace pkva
