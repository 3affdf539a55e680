// Host tile planner: validates one mixed prefill / decode / verify batch and decomposes it
// into fixed-shape tile tasks, then orders them for the launch.
//
// XY-Serve (arXiv 2412.18106), verdict page, core_discovery: the batch is broken into
// tile-level tasks (its Token-Table / Task-Table) that are then reordered to balance the
// cores; key_machinery: attention tiles are ordered by how much work they carry and dealt
// to the cores round-robin. Here the "cores" are the CTA slots of the B200 (SMs x resident
// CTAs), the task list is uploaded once per plan, and the hardware block scheduler deals
// the tasks out in list order, so heaviest-first order gives a longest-task-first schedule.
#include <math.h>
#include <stdio.h>

#include <algorithm>
#include <cstring>

#include "pkva.h"
#include "pkva_internal.h"

namespace pkva {

namespace {

constexpr int kMinSplitPages = 8;      // never split a unit into tasks below 128 keys
constexpr int kTasksPerSlot = 1;       // split long units down to about one task per CTA slot
// A row-split task's warps each run every page of the task, where a 16-row task's four warps
// share its pages: it gets a quarter of the pages of a 16-row task, so that its warps' page
// chains are as long as theirs, but no fewer than kMinWidePages (a task's set-up and the
// merge of its chunks' partials would outweigh shorter chains).
constexpr int kWideSplit = 4;
constexpr int kMinWidePages = 32;

int fail(std::string* err, int code, const char* fmt, long a = 0, long b = 0, long c = 0) {
    char buf[256];
    snprintf(buf, sizeof buf, fmt, a, b, c);
    if (err) *err = buf;
    return code;
}

}  // namespace

int build_host_plan(const PlanArgs& a, HostPlan* out, std::string* err) {
    HostPlan& p = *out;
    p = HostPlan();
    if (a.num_seqs < 0) return fail(err, PKVA_EINVAL, "num_seqs must be >= 0 (got %ld)", a.num_seqs);
    if (a.num_seqs > 0 && (!a.seq_lens || !a.query_lens || !a.mask_kind))
        return fail(err, PKVA_EINVAL, "seq_lens, query_lens and mask_kind must not be NULL");
    if (a.Hkv < 1 || a.Hq < 1 || a.Hq % a.Hkv != 0)
        return fail(err, PKVA_EINVAL, "num_q_heads (%ld) must be a positive multiple of num_kv_heads (%ld)",
                    a.Hq, a.Hkv);
    if (a.D != 64 && a.D != 128)
        return fail(err, PKVA_EUNSUPPORTED, "head_dim %ld not supported (64 or 128)", a.D);
    if (a.page_size != kPageSize)
        return fail(err, PKVA_EUNSUPPORTED, "page_size %ld not supported (16)", a.page_size);
    if (a.sm_scale != a.sm_scale) return fail(err, PKVA_EINVAL, "sm_scale is NaN");
    if (a.num_sms < 1 || a.ctas_per_sm < 1)
        return fail(err, PKVA_EINVAL, "num_sms and ctas_per_sm must be >= 1");

    p.num_seqs = a.num_seqs;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.D = a.D;
    p.bt_stride = a.bt_stride;
    p.num_pages = a.num_pages;
    p.scale = a.sm_scale > 0.f ? a.sm_scale : 1.0f / sqrtf((float)a.D);

    if (a.num_seqs > 0) {
        if (a.num_pages < 1) return fail(err, PKVA_EINVAL, "num_pages must be >= 1");
        if ((int64_t)a.num_pages * a.Hkv * kPageSize >= (int64_t(1) << 31))
            return fail(err, PKVA_EUNSUPPORTED, "cache too large: num_pages*Hkv*16 must be < 2^31");
    }

    // -- per-sequence records and tree masks ------------------------------------------
    int64_t q_acc = 0;
    int par_off = 0;
    for (int s = 0; s < a.num_seqs; ++s) {
        const int L = a.seq_lens[s], T = a.query_lens[s], mk = a.mask_kind[s];
        if (L < 1) return fail(err, PKVA_EINVAL, "seq_lens[%ld] = %ld must be >= 1", s, L);
        if (T < 1 || T > L)
            return fail(err, PKVA_EINVAL, "query_lens[%ld] = %ld must be in [1, seq_len = %ld]", s, T, L);
        if (mk != PKVA_CAUSAL && mk != PKVA_TREE)
            return fail(err, PKVA_EINVAL, "mask_kind[%ld] = %ld is not CAUSAL (0) or TREE (1)", s, mk);
        const int pages = (L + kPageSize - 1) / kPageSize;
        if (pages > a.bt_stride)
            return fail(err, PKVA_EINVAL, "sequence %ld needs %ld block-table entries; bt_stride is %ld",
                        s, pages, a.bt_stride);
        SeqInfo si{};
        si.seq_len = L;
        si.query_len = T;
        si.q_start = (int32_t)q_acc;
        si.mask_kind = mk;
        si.anc_off = -1;
        if (mk == PKVA_TREE) {
            if (T > kMaxTreeTokens)
                return fail(err, PKVA_EINVAL, "TREE sequence %ld has %ld draft tokens (max 64)", s, T);
            if (!a.parents) return fail(err, PKVA_EINVAL, "parents is NULL but sequence %ld is TREE", s);
            si.anc_off = (int32_t)p.anc.size();
            for (int i = 0; i < T; ++i) {
                const int par = a.parents[par_off + i];
                if (par < -1 || par >= i)
                    return fail(err, PKVA_EINVAL,
                                "parents of sequence %ld, node %ld = %ld: must be -1 or an earlier node",
                                s, i, par);
                uint64_t m = uint64_t(1) << i;
                if (par >= 0) m |= p.anc[si.anc_off + par];
                p.anc.push_back(m);
            }
            par_off += T;
        }
        p.seqs.push_back(si);
        q_acc += T;
        if (q_acc > (int64_t(1) << 31) / a.Hq)
            return fail(err, PKVA_EUNSUPPORTED, "too many query rows");

        // algorithmic work: every K and V element once; 4*D*Hq flops per allowed pair
        p.kv_bytes += (int64_t)L * a.Hkv * a.D * 2 /*K,V*/ * a.kv_elem_bytes;
        int64_t pairs = (int64_t)T * (L - T);
        if (mk == PKVA_CAUSAL) {
            pairs += (int64_t)T * (T + 1) / 2;
        } else {
            for (int i = 0; i < T; ++i) pairs += __builtin_popcountll(p.anc[si.anc_off + i]);
        }
        p.attn_flops += pairs * a.Hq * 4 * a.D;
    }
    p.total_q = (int)q_acc;

    // -- shared-prefix groups ------------------------------------------------------------
    std::vector<int> grp_of(a.num_seqs, -1);     // group of a sequence whose prefix is shared
    if (a.num_groups < 0) return fail(err, PKVA_EINVAL, "num_groups must be >= 0 (got %ld)", a.num_groups);
    if (a.num_groups > 0 && a.num_seqs > 0) {
        if (!a.prefix_group || !a.prefix_len)
            return fail(err, PKVA_EINVAL, "prefix_group and prefix_len must not be NULL when num_groups > 0");
        std::vector<int> first(a.num_groups, -1), last(a.num_groups, -1), count(a.num_groups, 0);
        for (int s = 0; s < a.num_seqs; ++s) {
            const int g = a.prefix_group[s];
            if (g < -1 || g >= a.num_groups)
                return fail(err, PKVA_EINVAL, "prefix_group[%ld] = %ld must be -1 or in [0, num_groups)", s, g);
            if (g < 0) continue;
            if (first[g] < 0) first[g] = s;
            last[g] = s;
            ++count[g];
        }
        for (int g = 0; g < a.num_groups; ++g) {
            const int P = a.prefix_len[g];
            if (P < 0 || P % kPageSize)
                return fail(err, PKVA_EINVAL, "prefix_len[%ld] = %ld must be a non-negative multiple of 16", g, P);
            if (first[g] < 0) continue;
            if (last[g] - first[g] + 1 != count[g])
                return fail(err, PKVA_EINVAL, "the sequences of prefix group %ld are not consecutive in the batch", g);
            for (int s = first[g]; s <= last[g]; ++s) {
                const SeqInfo& si = p.seqs[s];
                if (P > si.seq_len - si.query_len)
                    return fail(err, PKVA_EINVAL,
                                "prefix_len of group %ld (%ld) exceeds the committed prefix of sequence %ld", g, P, s);
            }
            if (P == 0) continue;
            if (a.D != 128 && a.kv_elem_bytes != 2)
                return fail(err, PKVA_EUNSUPPORTED,
                            "shared-prefix groups over FP8 caches need head_dim 128 (got %ld)", a.D);
            if (p.G > kPrefillTileM)
                return fail(err, PKVA_EUNSUPPORTED, "shared-prefix groups need at most 128 query heads per KV head");
            for (int s = first[g]; s <= last[g]; ++s) grp_of[s] = g;
        }
    }

    // keys each group's cascade tasks cover
    std::vector<int> glen;
    for (int g = 0; g < (a.num_seqs > 0 ? a.num_groups : 0); ++g) glen.push_back(a.prefix_len[g]);

    // -- prefill tiles: long causal chunks go to the tensor-core prefill kernel ---------
    std::vector<char> on_prefill(a.num_seqs, 0);
    // tensor-core tasks: head_dim 128, and 64 over bf16 caches (the FP8 staging copies are 128)
    const bool tc_ok = a.use_prefill_kernel && (a.D == 128 || a.kv_elem_bytes == 2);
    if (tc_ok) {
        for (int s = 0; s < a.num_seqs; ++s) {
            const SeqInfo& si = p.seqs[s];
            if (si.mask_kind != PKVA_CAUSAL || si.query_len < kPrefillMinTokens) continue;
            on_prefill[s] = 1;
            const int prefix = si.seq_len - si.query_len;
            const int cache_tiles = (prefix + kPrefillTileN - 1) / kPrefillTileN;
            const int ntt = (si.query_len + kPrefillTileM - 1) / kPrefillTileM;     // token tiles
            auto ntok_of = [&](int tt) { return std::min(kPrefillTileM, si.query_len - tt * kPrefillTileM); };
            // each tile needs keys up to its last row's own position (causal tile skipping)
            auto tiles_of = [&](int tt) {
                return (prefix + tt * kPrefillTileM + ntok_of(tt) + kPrefillTileN - 1) / kPrefillTileN;
            };
            auto tiles_app_of = [&](int tt) {
                return cache_tiles + (tt * kPrefillTileM + ntok_of(tt) - 1) / kPrefillTileN + 1;
            };
            auto add = [&](int h0, int tt0, int h1, int tt1) {    // tt1 < 0: no tile 1
                PrefillWork pw{};
                pw.seq = s;
                pw.q_head = h0;
                pw.tok0 = tt0 * kPrefillTileM;
                pw.ntok0 = ntok_of(tt0);
                pw.kv_tiles0 = tiles_of(tt0);
                pw.kv_tiles0_append = tiles_app_of(tt0);
                if (tt1 >= 0) {
                    pw.q_head1 = h1;
                    pw.tok1 = tt1 * kPrefillTileM;
                    pw.ntok1 = ntok_of(tt1);
                    pw.kv_tiles1 = tiles_of(tt1);
                    pw.kv_tiles1_append = tiles_app_of(tt1);
                } else {                                   // an absent tile loads (unused) rows past tile 0
                    pw.q_head1 = h0;
                    pw.tok1 = pw.tok0 + kPrefillTileM;
                }
                p.pwork.push_back(pw);
            };
            // pairs of query heads of one KV head on the same token tile; in an odd group the
            // last head pairs consecutive token tiles of its own
            for (int tt = 0; tt < ntt; ++tt)
                for (int kvh = 0; kvh < a.Hkv; ++kvh) {
                    const int h0 = kvh * p.G;
                    for (int i = 0; i + 1 < p.G; i += 2) add(h0 + i, tt, h0 + i + 1, tt);
                    if ((p.G & 1) && (tt & 1) == 0) add(h0 + p.G - 1, tt, h0 + p.G - 1, tt + 1 < ntt ? tt + 1 : -1);
                }
        }
        // heaviest first; equal work keeps (seq, token tile, KV head) order so that the query
        // heads of one GQA group run side by side and share their K/V tiles through L2
        std::stable_sort(p.pwork.begin(), p.pwork.end(), [](const PrefillWork& x, const PrefillWork& y) {
            return x.kv_tiles0 + x.kv_tiles1 > y.kv_tiles0 + y.kv_tiles1;
        });
    }

    // -- verify trees (and short causal chunks) of 17 to 128 packed rows per KV head run
    //    on the tensor cores: one cascade-style task per (sequence, KV head, chunk of
    //    kOwnTilesPerTask KV tiles) holds all of the unit's rows in one query tile and reads
    //    each key once for all of them (tree / causal masks on the tiles with the new tokens'
    //    keys); its halves interleave the KV tiles so that the tensor cores and the softmax
    //    overlap. bf16 caches only (FP8 would stage the whole sequence to bf16 first).
    //    Like the row-split rule below, only in a batch where such units hold at most half of
    //    the decode/verify pages: a tensor-core task takes a whole SM and streams its keys at
    //    about 40 GB/s, so it pays beside decode blocks that keep HBM busy, while a batch of
    //    such units alone ran faster as 16-row decode/verify tasks (measured on B200: the
    //    Qwen2-7B verify class 0.0614 against 0.0655 ms, the unified batch 0.170 against
    //    0.166 ms).
    std::vector<char> on_own(a.num_seqs, 0);
    if (a.self_cascade && tc_ok && a.D == 128 && a.kv_elem_bytes == 2 && p.G <= kPrefillTileM) {
        int64_t own_pages = 0, all_pages = 0;
        for (int s = 0; s < a.num_seqs; ++s) {
            if (on_prefill[s]) continue;
            const SeqInfo& si = p.seqs[s];
            const int64_t pg = (int64_t)(si.seq_len + kPageSize - 1) / kPageSize -
                               (grp_of[s] >= 0 ? glen[grp_of[s]] / kPageSize : 0);
            all_pages += pg;
            if (grp_of[s] >= 0 || si.query_len * p.G <= kDecodeRowsMax || si.query_len > kPrefillTileM / p.G ||
                si.seq_len < kOwnMinKeys)
                continue;
            on_own[s] = 1;
            own_pages += pg;
        }
        if (2 * own_pages > all_pages) std::fill(on_own.begin(), on_own.end(), 0);
    }

    // -- decode/verify units: (seq, kv head, chunk of packed rows) --------------------
    // A sequence of a shared-prefix group leaves its first prefix_len keys to the cascade
    // tasks: its units start at that page, and always merge partials.
    // cs: cascade splits (0: none). A row-split task covers several consecutive chunk units:
    // its first (lead) unit has wrows = the task's rows, the others wrows = 0; a plain unit
    // has wrows = rc. All chunks of a row-split task share its page range.
    struct Unit { int seq, kvh, rb, rc, pstart, pages, cs, wrows; };
    std::vector<Unit> units;
    // Row-split tasks pay off for units of three or more 16-row chunks (each page then read
    // once instead of three times) in a batch where such units are a minority of the
    // decode/verify pages: there the other tasks keep the SMs busy while the row-split
    // tasks' warps each run all of their pages; a batch made mostly of such units keeps the
    // 16-row tasks, whose four warps share a unit's pages (measured on B200: a verify-only
    // batch took 2.4x longer with row-split tasks, the mixed batch 9 % less time).
    bool wide = a.wide_tasks && a.kv_elem_bytes == 2;
    if (wide) {
        int64_t wide_pages = 0, all_pages = 0;
        for (int s = 0; s < a.num_seqs; ++s) {
            if (on_prefill[s] || on_own[s]) continue;
            const SeqInfo& si = p.seqs[s];
            const int64_t pg = (int64_t)(si.seq_len + kPageSize - 1) / kPageSize -
                               (grp_of[s] >= 0 ? glen[grp_of[s]] / kPageSize : 0);
            all_pages += pg;
            if (si.query_len * p.G > 2 * kDecodeRowsMax) wide_pages += pg;
        }
        wide = 2 * wide_pages <= all_pages;
    }
    std::vector<int> unit_base(a.num_seqs, -1);     // index of (s, head 0, chunk 0) in units
    std::vector<char> on_cascade(a.num_seqs, 0);
    int64_t total_pages = 0;
    int max_rc = 0;
    for (int s = 0; s < a.num_seqs; ++s) {
        if (on_prefill[s]) continue;
        const SeqInfo& si = p.seqs[s];
        const int rows = si.query_len * p.G;
        const int g = grp_of[s];
        if (on_own[s]) {
            // tensor-core rows: one unit per 16-row chunk (split slots for the KV chunks; none
            // when one task covers all keys and writes the rows itself), no decode/verify task
            const int tiles = (si.seq_len + kPrefillTileN - 1) / kPrefillTileN;
            int cs = (tiles + kOwnTilesPerTask - 1) / kOwnTilesPerTask;
            if (cs == 1) cs = 0;
            unit_base[s] = (int)units.size();
            for (int h = 0; h < a.Hkv; ++h)
                for (int rb = 0; rb < rows; rb += kDecodeRowsMax) {
                    const int rc = std::min(kDecodeRowsMax, rows - rb);
                    units.push_back({s, h, rb, rc, 0, 0, cs, rc});
                }
            continue;
        }
        const int pstart = g >= 0 ? glen[g] / kPageSize : 0;
        const int cs = g >= 0 ? (glen[g] + kPrefillTileN * kCascadeTilesPerTask - 1) /
                                    (kPrefillTileN * kCascadeTilesPerTask)
                              : 0;
        on_cascade[s] = g >= 0;
        p.seqs[s].shared_len = g >= 0 ? glen[g] : 0;
        unit_base[s] = (int)units.size();
        // keys past the last row's own position are masked for every row of a task (causal
        // and tree alike), so the task never loads them
        auto pages_to = [&](int last_row) {
            const int kend = si.seq_len - si.query_len + last_row / p.G + 1;
            return (kend + kPageSize - 1) / kPageSize;
        };
        for (int h = 0; h < a.Hkv; ++h) {
            for (int tb = 0; tb < rows; tb += wide ? kWideRowsMax : kDecodeRowsMax) {
                const int tr = std::min(wide ? kWideRowsMax : kDecodeRowsMax, rows - tb);
                if (tr <= 2 * kDecodeRowsMax) {          // one or two 16-row tasks
                    for (int rb = tb; rb < tb + tr; rb += kDecodeRowsMax) {
                        const int rc = std::min(kDecodeRowsMax, tb + tr - rb);
                        const int pages = pages_to(rb + rc - 1);
                        units.push_back({s, h, rb, rc, pstart, pages, cs, rc});
                        total_pages += pages - pstart;
                        max_rc = std::max(max_rc, rc);
                    }
                    continue;
                }
                // one row-split task: its 16-row chunks, the whole row range's pages
                const int pages = pages_to(tb + tr - 1);
                for (int rb = tb; rb < tb + tr; rb += kDecodeRowsMax)
                    units.push_back({s, h, rb, std::min(kDecodeRowsMax, tb + tr - rb), pstart, pages, cs,
                                     rb == tb ? tr : 0});
                total_pages += pages - pstart;
            }
        }
    }
    // algorithmic bytes: a shared prefix is one set of keys, counted once per group
    if (!glen.empty()) {
        std::vector<char> counted(glen.size(), 0);
        for (int s = 0; s < a.num_seqs; ++s) {
            if (!on_cascade[s]) continue;
            const int g = grp_of[s];
            const int64_t per_key = (int64_t)a.Hkv * a.D * 2 * a.kv_elem_bytes;
            p.kv_bytes -= (int64_t)glen[g] * per_key;
            if (!counted[g]) p.kv_bytes += (int64_t)glen[g] * per_key;
            counted[g] = 1;
        }
    }
    p.decode_rows = max_rc <= 4 ? 4 : (max_rc <= 8 ? 8 : 16);
    if (units.empty()) p.decode_rows = 4;

    // -- split long units so the grid has ~kTasksPerSlot tasks per CTA slot -------------
    // When the per-task page cap forces more than one task per slot over FP8 caches, the
    // target is set so that the tasks fill whole waves of slots: the FP8 body converts
    // codes at about twice the instructions per byte, so a last wave only partly filled
    // leaves HBM idle. The bf16 body keeps HBM busy with a partial last wave, and there
    // the fewer, longer tasks measured faster.
    const int64_t per_wave = (int64_t)a.num_sms * a.ctas_per_sm * kTasksPerSlot;
    const int64_t waves =
        a.kv_elem_bytes == 1 ? std::max<int64_t>(1, (total_pages + per_wave * kDecodeMaxPages - 1) /
                                                        (per_wave * kDecodeMaxPages))
                             : 1;
    int64_t target = (total_pages + per_wave * waves - 1) / (per_wave * waves);
    target = std::max<int64_t>(target, kMinSplitPages);
    target = std::min<int64_t>(target, kDecodeMaxPages);
    std::vector<int> unit_id_of(units.size(), -1);
    std::vector<int> unit_ns(units.size(), 0);
    for (size_t ui = 0; ui < units.size(); ++ui) {
        const Unit& u = units[ui];
        if (u.wrows == 0) continue;           // a later chunk of a row-split task: done with its lead
        const int own = u.pages - u.pstart;
        const int nchunks = (u.wrows + kDecodeRowsMax - 1) / kDecodeRowsMax;
        // nearest whole number of target-sized tasks (rounding up made near-target units two
        // half-size tasks), never more pages per task than the staged block-table slice holds
        const int64_t per_task = nchunks > 1 ? std::max<int64_t>(target / kWideSplit, kMinWidePages) : target;
        const int ns = on_own[u.seq] ? 0          // tensor-core rows: only cascade-style tasks
                                     : std::max<int>(std::max<int>(1, (int)((own + per_task / 2) / per_task)),
                                                     (own + kDecodeMaxPages - 1) / kDecodeMaxPages);
        int unit_id = -1;                     // the lead chunk's; chunk c has unit_id + c
        for (int c = 0; c < nchunks; ++c) {
            const Unit& uc = units[ui + c];
            unit_ns[ui + c] = ns;
            int id = -1;
            if (ns > 1 || uc.cs > 0) {
                id = (int)p.units.size();
                SplitUnit su{};
                su.slot_base = p.num_slots;
                su.num_splits = ns + uc.cs;
                su.arrivals = ns;             // cascade tasks add theirs below
                su.seq = uc.seq;
                su.kv_head = uc.kvh;
                su.row_begin = uc.rb;
                su.row_count = uc.rc;
                p.units.push_back(su);
                p.num_slots += ns + uc.cs;
            }
            unit_id_of[ui + c] = id;
            if (c == 0) unit_id = id;
        }
        for (int k = 0; k < ns; ++k) {
            DecodeWork w{};
            w.seq = u.seq;
            w.kv_head = u.kvh;
            w.row_begin = u.rb;
            w.row_count = u.wrows;
            w.page_begin = u.pstart + (int)((int64_t)own * k / ns);
            w.page_end = u.pstart + (int)((int64_t)own * (k + 1) / ns);
            w.unit = unit_id;
            w.split = unit_id >= 0 ? k : -1;
            p.dwork.push_back(w);
        }
    }

    // -- shared-prefix (cascade) tasks: per group, per run of consecutive decode-path
    //    members (their q rows are contiguous), per KV head: tiles of floor(128 / G) tokens
    //    x G heads, two tiles per task, the prefix split into chunks of tiles ---------------
    p.cascade_tok = kPrefillTileM / p.G;
    if (!glen.empty()) {
        const int TOK = p.cascade_tok;
        auto seq_of_token = [&](int tok) {
            int lo = 0, hi = a.num_seqs - 1;       // last s with q_start <= tok
            while (lo < hi) {
                const int mid = (lo + hi + 1) / 2;
                if (p.seqs[mid].q_start <= tok) lo = mid; else hi = mid - 1;
            }
            return lo;
        };
        int s = 0;
        while (s < a.num_seqs) {
            if (!on_cascade[s]) { ++s; continue; }
            const int g = grp_of[s];
            int e = s;
            while (e + 1 < a.num_seqs && on_cascade[e + 1] && grp_of[e + 1] == g) ++e;
            const int run_t0 = p.seqs[s].q_start;
            const int run_t1 = p.seqs[e].q_start + p.seqs[e].query_len;
            const int tiles = (glen[g] + kPrefillTileN - 1) / kPrefillTileN;
            const int cs = units[unit_base[s]].cs;
            for (int h = 0; h < a.Hkv; ++h) {
                for (int t0 = run_t0; t0 < run_t1; t0 += 2 * TOK) {
                    const int ntok = std::min(2 * TOK, run_t1 - t0);
                    for (int k = 0; k < cs; ++k) {
                        CascadeWork cw{};
                        cw.lead_seq = s;
                        cw.kv_head = h;
                        cw.tok0 = t0;
                        cw.ntok = ntok;
                        cw.tile_begin = (int)((int64_t)tiles * k / cs);
                        cw.tile_end = (int)((int64_t)tiles * (k + 1) / cs);
                        cw.unit_off = (int)p.cunits.size();
                        int last_unit = -1;
                        for (int b = 0; b < 2; ++b) {
                            for (int r = 0; r < kPrefillTileM; ++r) {
                                const int tl = b * TOK + r / p.G;
                                int entry = -1;
                                if (r < TOK * p.G && tl < ntok) {
                                    const int tok = t0 + tl;
                                    const int sq = seq_of_token(tok);
                                    const int pr = (tok - p.seqs[sq].q_start) * p.G + r % p.G;
                                    const int chunks = (p.seqs[sq].query_len * p.G + kDecodeRowsMax - 1) /
                                                       kDecodeRowsMax;
                                    const int ui = unit_base[sq] + h * chunks + pr / kDecodeRowsMax;
                                    const int uid = unit_id_of[ui];
                                    entry = (p.units[uid].slot_base + unit_ns[ui] + k) * kDecodeRowsMax +
                                            pr % kDecodeRowsMax;
                                    if (uid != last_unit) {      // rows of one unit are adjacent
                                        p.cunits.push_back(uid);
                                        p.units[uid].arrivals += 1;
                                        last_unit = uid;
                                    }
                                }
                                p.crowmap.push_back(entry);
                            }
                        }
                        cw.unit_cnt = (int)p.cunits.size() - cw.unit_off;
                        p.cwork.push_back(cw);
                    }
                }
            }
            s = e + 1;
        }
    }
    // -- tensor-core verify tasks (see on_own): all of a unit's rows in tile 0, its KV tiles
    //    split into chunks of kOwnTilesPerTask --------------------------------------------
    for (int s = 0; s < a.num_seqs; ++s) {
        if (!on_own[s]) continue;
        const SeqInfo& si = p.seqs[s];
        const int rows = si.query_len * p.G;
        const int chunks = (rows + kDecodeRowsMax - 1) / kDecodeRowsMax;
        const int tiles = (si.seq_len + kPrefillTileN - 1) / kPrefillTileN;
        const int cs = std::max(1, units[unit_base[s]].cs);
        const bool direct = units[unit_base[s]].cs == 0;       // one task: it writes the rows
        for (int h = 0; h < a.Hkv; ++h) {
            const int ub = unit_base[s] + h * chunks;
            for (int k = 0; k < cs; ++k) {
                CascadeWork cw{};
                cw.lead_seq = s;
                cw.kv_head = h;
                cw.tok0 = si.q_start;
                cw.ntok = si.query_len;
                cw.tile_begin = (int)((int64_t)tiles * k / cs);
                cw.tile_end = (int)((int64_t)tiles * (k + 1) / cs);
                cw.unit_off = (int)p.cunits.size();
                cw.unit_cnt = direct ? 0 : chunks;
                cw.own = direct ? 2 : 1;
                for (int c = 0; c < cw.unit_cnt; ++c) {
                    p.cunits.push_back(unit_id_of[ub + c]);
                    p.units[unit_id_of[ub + c]].arrivals += 1;
                }
                for (int r = 0; r < 2 * kPrefillTileM; ++r)
                    p.crowmap.push_back(!direct && r < rows
                                            ? (p.units[unit_id_of[ub + r / kDecodeRowsMax]].slot_base + k) *
                                                      kDecodeRowsMax + r % kDecodeRowsMax
                                            : -1);
                p.cwork.push_back(cw);
            }
        }
    }
    // FP8 caches: the tensor-core tasks read a bf16 copy of the pages they use: all pages of
    // a sequence that runs as prefill tasks, the shared pages of a cascade run's lead sequence
    // (whose block-table row supplies the shared keys to its cascade tasks)
    if (a.kv_elem_bytes == 1) {
        std::vector<int> stage_pages(a.num_seqs, 0);
        for (int s = 0; s < a.num_seqs; ++s)
            if (on_prefill[s]) stage_pages[s] = (p.seqs[s].seq_len + kPageSize - 1) / kPageSize;
        for (const CascadeWork& cw : p.cwork)
            stage_pages[cw.lead_seq] = glen[grp_of[cw.lead_seq]] / kPageSize;
        int stride = 0;
        int64_t n = 0;
        for (int s = 0; s < a.num_seqs; ++s) {
            stride = std::max(stride, stage_pages[s]);
            n += stage_pages[s];
        }
        if (n * a.Hkv * kPageSize >= (int64_t(1) << 31))
            return fail(err, PKVA_EUNSUPPORTED, "FP8 tensor-core staging too large: %ld pages", (long)n);
        if (n > 0) {
            p.stage_stride = stride;
            p.num_stage_pages = (int)n;
            p.stage_bt.assign((size_t)a.num_seqs * stride, -1);
            p.stage_src.reserve(2 * (size_t)n);
            int next = 0;
            for (int s = 0; s < a.num_seqs; ++s) {
                for (int lp = 0; lp < stage_pages[s]; ++lp) {
                    p.stage_bt[(size_t)s * stride + lp] = next++;
                    p.stage_src.push_back(s);
                    p.stage_src.push_back(lp);
                }
            }
        }
    }

    // heaviest first; ties keep (seq, head, chunk) order so chunks of one head stay adjacent
    // (a row-split task weighs its pages kWideSplit times: each of its warps runs every page)
    auto task_cost = [](const DecodeWork& w) {
        return (w.page_end - w.page_begin) * (w.row_count > kDecodeRowsMax ? kWideSplit : 1);
    };
    std::stable_sort(p.dwork.begin(), p.dwork.end(), [&](const DecodeWork& x, const DecodeWork& y) {
        return task_cost(x) > task_cost(y);
    });

    // -- one launch order. Shared-prefix cascade tasks go first: few, long, and every unit of
    //    their rows waits for them, so the units' own decode tasks tend to arrive last and do
    //    the merges, spread over many blocks. The other tensor-core tasks (prefill tiles and
    //    tensor-core verify tasks, heaviest first by the KV tiles each query tile runs) and
    //    the decode tasks (heaviest first) are merged in proportion, so tensor-core blocks
    //    (latency) run beside decode blocks (HBM) from start to end instead of one kind
    //    forming the tail; the tensor-core list runs 1.25x ahead of its share, so that its
    //    long blocks are not the last to finish (measured on the Qwen2-7B-shaped unified
    //    batch: 0.1638 against 0.166 ms in plain proportion; 1.75x ahead, 0.172 ms). Decode
    //    tasks go three to a block, neighbours in the sorted list.
    std::vector<int32_t> tc;                  // block entries of the tensor-core list
    std::vector<int> tc_cost;
    for (size_t i = 0; i < p.pwork.size(); ++i) {
        tc.push_back((int32_t)i);
        tc_cost.push_back(p.pwork[i].kv_tiles0 + p.pwork[i].kv_tiles1);
    }
    for (size_t i = 0; i < p.cwork.size(); ++i) {
        const int32_t e = (int32_t)(p.pwork.size() + i);
        if (!p.cwork[i].own) {
            p.order.push_back(e);
            continue;
        }
        tc.push_back(e);
        tc_cost.push_back(p.cwork[i].tile_end - p.cwork[i].tile_begin);
    }
    std::vector<int> tci(tc.size());
    for (size_t i = 0; i < tc.size(); ++i) tci[i] = (int)i;
    std::stable_sort(tci.begin(), tci.end(), [&](int x, int y) { return tc_cost[x] > tc_cost[y]; });
    const int np = (int)tc.size();
    const int nd = (int)((p.dwork.size() + kDecTasksPerBlock - 1) / kDecTasksPerBlock);
    int ip = 0, id = 0;
    while (ip < np || id < nd) {
        // take from the list that is further behind in its share of the launch
        const bool take_p = id >= nd || (ip < np && (int64_t)ip * nd * 4 <= (int64_t)(id + 1) * np * 5);
        if (take_p)
            p.order.push_back(tc[tci[ip++]]);
        else
            p.order.push_back(-1 - id++);
    }
    return PKVA_OK;
}

}  // namespace pkva

namespace pkva {
void set_last_error(const std::string& msg);   // defined with the rest of the C ABI
}

extern "C" int attn_plan_inspect(int num_seqs, const int32_t* seq_lens, const int32_t* query_lens,
                                 int bt_stride, int num_pages, const int32_t* mask_kind,
                                 const int32_t* parents, int num_q_heads, int num_kv_heads,
                                 int head_dim, int page_size, const int32_t* prefix_group,
                                 const int32_t* prefix_len, int num_groups, int num_sms, int ctas_per_sm,
                                 pkva_work_desc* items, int max_items, int* num_items) {
    using namespace pkva;
    PlanArgs a{num_seqs, seq_lens, query_lens, bt_stride, num_pages, mask_kind, parents,
               num_q_heads, num_kv_heads, head_dim, page_size, 0.f, num_sms, ctas_per_sm};
    a.prefix_group = prefix_group;
    a.prefix_len = prefix_len;
    a.num_groups = num_groups;
    HostPlan hp;
    std::string err;
    int rc = build_host_plan(a, &hp, &err);
    if (rc != PKVA_OK) {
        set_last_error(err);
        return rc;
    }
    // prefill tasks are listed one entry per query tile (a task holds one or two)
    int np = 0;
    for (const PrefillWork& w : hp.pwork) np += w.ntok1 > 0 ? 2 : 1;
    const int nc = (int)hp.cwork.size();
    const int n = np + nc + (int)hp.dwork.size();
    if (num_items) *num_items = n;
    if (!items) return PKVA_OK;
    if (max_items < n) {
        set_last_error("attn_plan_inspect: max_items is smaller than the number of tasks");
        return PKVA_EINVAL;
    }
    int ip = nc;
    for (const PrefillWork& w : hp.pwork) {      // prefill tiles after the cascade tasks
        const SeqInfo& si = hp.seqs[w.seq];
        for (int b = 0; b < (w.ntok1 > 0 ? 2 : 1); ++b) {
            const int h = b ? w.q_head1 : w.q_head, t0 = b ? w.tok1 : w.tok0, nt = b ? w.ntok1 : w.ntok0;
            pkva_work_desc d;
            d.kind = 1;
            d.seq = w.seq;
            d.kv_head = h / hp.G;
            d.q_head = h;
            d.row_begin = t0;
            d.row_count = nt;
            d.key_begin = 0;
            d.key_end = std::min(si.seq_len - si.query_len + t0 + nt, si.seq_len);
            d.split = -1;
            d.num_splits = 1;
            items[ip++] = d;
        }
    }
    for (int i = 0; i < nc; ++i) {      // shared-prefix (cascade) tasks first, as in the launch
        const CascadeWork& w = hp.cwork[i];
        // keys the task's unit covers: the shared prefix, or (tensor-core verify rows) the
        // whole sequence
        const int P = w.own ? hp.seqs[w.lead_seq].seq_len : hp.seqs[w.lead_seq].shared_len;
        const int tiles = (P + kPrefillTileN - 1) / kPrefillTileN;
        const int cs = w.own ? (tiles + kOwnTilesPerTask - 1) / kOwnTilesPerTask
                             : (P + kPrefillTileN * kCascadeTilesPerTask - 1) / (kPrefillTileN * kCascadeTilesPerTask);
        int k = 0;
        while (k < cs && (int)((int64_t)tiles * k / cs) != w.tile_begin) ++k;
        pkva_work_desc d;
        d.kind = 2;
        d.seq = w.lead_seq;
        d.kv_head = w.kv_head;
        d.q_head = -1;
        d.row_begin = w.tok0;
        d.row_count = w.ntok;
        d.key_begin = w.tile_begin * kPrefillTileN;
        d.key_end = std::min(w.tile_end * kPrefillTileN, P);
        d.split = k;
        d.num_splits = cs;
        items[i] = d;
    }
    for (int i = np + nc; i < n; ++i) {
        const DecodeWork& w = hp.dwork[i - np - nc];
        const SeqInfo& si = hp.seqs[w.seq];
        pkva_work_desc d;
        d.kind = 0;
        d.seq = w.seq;
        d.kv_head = w.kv_head;
        d.q_head = -1;
        d.row_begin = w.row_begin;
        d.row_count = w.row_count;
        d.key_begin = w.page_begin * kPageSize;
        d.key_end = std::min(w.page_end * kPageSize, si.seq_len);
        d.split = w.split;
        d.num_splits = w.unit >= 0 ? hp.units[w.unit].num_splits : 1;
        items[i] = d;
    }
    set_last_error("");
    return PKVA_OK;
}
