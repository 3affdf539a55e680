// The prefill task body (see the description where this file is included). Included twice
// by pkva_prefill_body.cuh: as prefill_task (PKVA_PREFILL_RS 0) and as prefill_task_rs
// (PKVA_PREFILL_RS 1), the same body with the block's registers split between its
// warpgroups (setmaxnreg), which kernels with decode blocks beside the tensor-core tasks use.
// No include guard: it is meant to be included once per variant.

template <int D>
__device__ __forceinline__ void PKVA_PREFILL_TASK(const PrefillParams& p, int task, const CUtensorMap& tmQ,
                                             const CUtensorMap& tmK, const CUtensorMap& tmV,
                                             const CUtensorMap& tmKn, const CUtensorMap& tmVn,
                                             const CUtensorMap& tmQc, uint32_t tmem, uint8_t* sm) {
    using L = Lay<D>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool cascade = task >= p.num_prefill;
    const int ci = task - p.num_prefill;
    PrefillWork w{};
    CascadeWork cw{};
    if (cascade) {
        cw = p.cwork[ci];
        w.seq = cw.lead_seq;
        w.tok0 = cw.tok0;
        w.ntok0 = cw.ntok;
    } else {
        w = p.work[task];
    }
    const SeqInfo si = p.seqs[w.seq];
    const Bars B = bars_at<D>(sm);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffFlag);
    const bool append = p.append != 0 && !cascade;
    const int TOK = p.cascade_tok;                      // cascade: tokens per query tile
    const bool il = cascade && cw.ntok <= TOK;          // one query tile, KV tiles interleaved
    const int ncas = cw.tile_end - cw.tile_begin;
    const int n0 = il ? (ncas + 1) / 2 : cascade ? ncas : append ? w.kv_tiles0_append : w.kv_tiles0;
    const int n1 = il ? ncas / 2 : cascade ? (cw.ntok > TOK ? ncas : 0) : append ? w.kv_tiles1_append : w.kv_tiles1;
    const int nmax = il ? ncas : (n0 > n1 ? n0 : n1);   // KV tiles loaded, in order
    const int jbase = cascade ? cw.tile_begin : 0;     // first KV tile (of 128 keys) of the task
    const int kvh = cascade ? cw.kv_head : w.q_head / p.G;
    const int prefix = si.seq_len - si.query_len;
    const int nc = append ? (prefix + kPrefillTileN - 1) / kPrefillTileN : nmax;   // tiles read from the cache
    // cache keys that hold data: the shared prefix (cascade), the committed prefix
    // (append), the whole sequence (otherwise)
    // own: a tensor-core verify task, the rows of one sequence over its own keys (masked)
    const bool own = cascade && cw.own != 0;
    const int key_limit = own ? si.seq_len : cascade ? si.shared_len : append ? prefix : si.seq_len;

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
            mbar_init(&B.o_ready[b], 1);
        }
        mbar_init(B.mma_done, 1);
        mbar_init(B.v_fix, 1);
        mbar_init(B.k_fix, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

#if PKVA_PREFILL_RS
    // each warpgroup enters its roles through a branch of its own, behind its own register
    // count: the producer / MMA / append warpgroup gives registers to the two softmax
    // warpgroups (3 x 128 threads x 168 = 2 x 128 x 192 + 128 x 120)
    if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;\n" ::: "memory");
#endif
    if (warp == kWarpKProd || warp == kWarpVProd) {
        // ------------------ TMA producers: warp 8 loads Q and K, warp 10 loads V ------------
        // lane 0 issues the loads; the whole warp patches a tile before releasing it
        const bool is_k = warp == kWarpKProd;
        const int32_t* btrow = p.block_table + (int64_t)w.seq * p.bt_stride;
        // the cache page holding key_limit has stale rows from key_limit on (when it is
        // not page-aligned): the V tile with that page is zeroed there before its PV
        const int fix_tile = (key_limit % kPageSize) ? key_limit / kPageSize / 8 - jbase : -1;
        if (lane == 0) {
            fence_proxy_async_smem();              // the previous task's generic accesses come first
            if (is_k && cascade) {
                // G heads x TOK tokens per tile: rows (token, head) in the tile's first
                // G * TOK rows, the same 128-byte rows as a one-head box
                prefetch_tensormap(&tmQc);
                prefetch_tensormap(&tmK);
                const int nq = il ? 1 : 2;                 // interleaved: both halves read Q tile 0
                mbar_arrive_expect_tx(B.q_full, (uint32_t)L::kHalves * (uint32_t)nq * (uint32_t)(p.G * TOK) * 128u);
                for (int b = 0; b < nq; ++b)
#pragma unroll
                    for (int h = 0; h < L::kHalves; ++h)
                        tma_load_3d(sm + L::kOffQ + b * L::kTileBytes + h * kHalfBytes, &tmQc, B.q_full, h * 64,
                                    kvh * p.G, cw.tok0 + b * TOK);
            } else if (is_k) {
                prefetch_tensormap(&tmQ);
                prefetch_tensormap(&tmK);
                if (append) prefetch_tensormap(&tmKn);
                mbar_arrive_expect_tx(B.q_full, 2 * L::kTileBytes);
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int h = 0; h < L::kHalves; ++h)
                        tma_load_3d(sm + L::kOffQ + b * L::kTileBytes + h * kHalfBytes, &tmQ, B.q_full, h * 64,
                                    b ? w.q_head1 : w.q_head, si.q_start + (b ? w.tok1 : w.tok0));
            } else {
                prefetch_tensormap(&tmV);
                if (append) prefetch_tensormap(&tmVn);
            }
        }
        const int NSt = is_k ? kNK : kNV;
        uint64_t* full = is_k ? B.k_full : B.v_full;
        uint64_t* empty = is_k ? B.k_empty : B.v_empty;
        uint64_t* fixbar = is_k ? B.k_fix : B.v_fix;
        uint8_t* base = sm + (is_k ? L::kOffK : L::kOffV);
        int nfix = 0;                                  // phases of fixbar used
        for (int j = 0; j < nmax; ++j) {
            const int st = j % NSt;
            if (j >= NSt &&
                !__all_sync(0xffffffffu, wait_or_abort(&empty[st], ((j / NSt) - 1) & 1, p.err, abort_flag)))
                break;
            uint8_t* dst = base + st * L::kTileBytes;
            if (j >= nc) {
                // new tokens [128 (j - nc), +128) of the chunk, straight from the input
                if (lane == 0) {
                    const int row0 = si.q_start + (j - nc) * kPrefillTileN;
                    mbar_arrive_expect_tx(&full[st], L::kTileBytes);
#pragma unroll
                    for (int h = 0; h < L::kHalves; ++h)
                        tma_load_3d(dst + h * kHalfBytes, is_k ? &tmKn : &tmVn, &full[st], h * 64, kvh, row0);
                }
                continue;
            }
            int rows[8];
            tile_rows(p, btrow, key_limit, kvh, jbase + j, rows);
            // a tensor-core verify task under fused append: the new tokens' keys are not in
            // the cache yet, their rows come from the dense input
            const int kb = (jbase + j) * kPrefillTileN;
            const bool patch = own && p.append && kb + kPrefillTileN > prefix && kb < si.seq_len;
            const bool zero = !is_k && j == fix_tile;
            if (!patch && !zero) {
                load_tile<D>(dst, is_k ? &tmK : &tmV, &full[st], rows, lane);
                continue;
            }
            load_tile<D>(dst, is_k ? &tmK : &tmV, fixbar, rows, lane);
            if (!__all_sync(0xffffffffu, wait_or_abort(fixbar, nfix & 1, p.err, abort_flag))) break;
            ++nfix;
            if (patch) {
                const int k0 = max(prefix, kb), k1 = min(si.seq_len, kb + kPrefillTileN);
                const __nv_bfloat16* src = is_k ? p.k_new : p.v_new;
                for (int idx = lane; idx < (k1 - k0) * (D / 8); idx += 32) {
                    const int key = k0 + idx / (D / 8), c = idx % (D / 8), r = key - kb;   // chunk c: half c / 8
                    const uint4 v = *reinterpret_cast<const uint4*>(
                        src + ((int64_t)(si.q_start + key - prefix) * p.Hkv + kvh) * D + c * 8);
                    *reinterpret_cast<uint4*>(dst + (c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v;
                }
            }
            if (zero) {
                const int pg = (key_limit / kPageSize) % 8, r0 = key_limit % kPageSize;
                for (int idx = lane; idx < (kPageSize - r0) * (D / 8); idx += 32) {
                    const int r = r0 + idx / (D / 8), c = idx % (D / 8);
                    *reinterpret_cast<uint4*>(dst + (c >> 3) * kHalfBytes + (pg * kPageSize + r) * 128 + (c & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_proxy_async_smem();                  // every lane's writes, before the MMAs read them
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[st]);
        }
        // drain: the last stages' release arrives (from tcgen05.commit) must have landed
        // before the task ends and its barriers are invalidated and reused
        for (int j = nmax > NSt ? nmax - NSt : 0; j < nmax; ++j)
            if (!__all_sync(0xffffffffu, wait_or_abort(&empty[j % NSt], (j / NSt) & 1, p.err, abort_flag))) break;
    } else if (warp == kWarpMma) {
        // ------------------------------ MMA issuer -------------------------------------------
        if (lane == 0) {
            const uint32_t q_base = smem_addr(sm + L::kOffQ);
            const uint32_t k_base = smem_addr(sm + L::kOffK);
            const uint32_t v_base = smem_addr(sm + L::kOffV);
            auto issue_qk = [&](int b, int j) {           // S_b = Q_b K_j^T (interleaved: Q_0)
                const int st = j % kNK;
                const uint32_t d = tmem + kColS + b * 128;
                const uint32_t qt = q_base + (il ? 0 : b) * L::kTileBytes;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kHalfBytes + (ks & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(qt + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(k_base + st * L::kTileBytes + off, 16, 1024);
                    tc_mma_ss(d, ad, bd, kIdescQK, ks > 0);
                }
                tc_commit(&B.s_full[b]);
            };
            auto issue_pv = [&](int b, int j, bool acc) {   // O_b (+)= P_b V_j
                const int st = j % kNV;
                const uint32_t pcol = tmem + kColS + b * 128;
#pragma unroll
                for (int ks = 0; ks < kPrefillTileN / 16; ++ks) {
                    const uint64_t bd = smem_desc_sw128(v_base + st * L::kTileBytes + ks * 2048, kHalfBytes, 1024);
                    tc_mma_ts(tmem + kColO + b * D, pcol + ks * 8, bd, L::kIdescPV, (acc || ks > 0) ? 1u : 0u);
                }
            };
            bool ok = wait_or_abort(B.q_full, 0, p.err, abort_flag) &&
                      wait_or_abort(&B.k_full[0], 0, p.err, abort_flag);
            if (ok && il) {
                // interleaved: S_0 of KV tile 0 and S_1 of KV tile 1 first; then per KV tile j
                // (half b = j % 2): PV of j, and QK^T of b's next tile j + 2
                tc_fence_after();
                issue_qk(0, 0);
                tc_commit(&B.k_empty[0]);
                if (n1 > 0) {
                    ok = wait_or_abort(&B.k_full[1], 0, p.err, abort_flag);
                    if (ok) {
                        tc_fence_after();
                        issue_qk(1, 1);
                        tc_commit(&B.k_empty[1]);
                    }
                }
                for (int j = 0; ok && j < nmax; ++j) {
                    const int b = j & 1, i = j >> 1, vst = j % kNV;
                    if (!wait_or_abort(&B.v_full[vst], (j / kNV) & 1, p.err, abort_flag) ||
                        !spin_or_abort(&B.p_full[b], i & 1, p.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(b, j, i > 0);
                    if (i == (b ? n1 : n0) - 1) tc_commit(&B.o_ready[b]);
                    tc_commit(&B.v_empty[vst]);
                    if (j + 2 < nmax) {
                        const int kst = (j + 2) % kNK;
                        if (!wait_or_abort(&B.k_full[kst], ((j + 2) / kNK) & 1, p.err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_qk(b, j + 2);
                        tc_commit(&B.k_empty[kst]);
                    }
                }
            } else if (ok) {
                tc_fence_after();
                if (n0 > 0) issue_qk(0, 0);
                if (n1 > 0) issue_qk(1, 0);
                tc_commit(&B.k_empty[0]);
            }
            for (int j = 0; ok && !il && j < nmax; ++j) {
                const int vst = j % kNV;
                bool vwaited = false, kwaited = false;
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int nb = b ? n1 : n0;
                    if (j >= nb) continue;
                    if (!vwaited) {
                        if (!wait_or_abort(&B.v_full[vst], (j / kNV) & 1, p.err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        vwaited = true;
                    }
                    if (!spin_or_abort(&B.p_full[b], j & 1, p.err, abort_flag)) {   // critical path
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(b, j, j > 0);
                    if (j == nb - 1) tc_commit(&B.o_ready[b]);
                    if (j + 1 < nb) {
                        if (!kwaited) {
                            if (!wait_or_abort(&B.k_full[(j + 1) % kNK], ((j + 1) / kNK) & 1, p.err, abort_flag)) {
                                ok = false;
                                break;
                            }
                            kwaited = true;
                            tc_fence_after();
                        }
                        issue_qk(b, j + 1);
                    }
                }
                if (!ok) break;
                tc_commit(&B.v_empty[vst]);
                if (kwaited) tc_commit(&B.k_empty[(j + 1) % kNK]);
            }
            // every MMA this thread issued must finish before TMEM is released
            tc_commit(B.mma_done);
            mbar_wait_bounded(B.mma_done, 0, p.err, PKVA_DEVERR_TIMEOUT);
        }
#if PKVA_PREFILL_RS
    } else if (own && p.append && warp == kPThreads / 32) {
        // ------------------- warp 11: a tensor-core verify task's cache writes ----------------
        // the task with the unit's last KV tiles writes the sequence's new rows of its KV head
        // (no other task reads those cache slots: any task whose tiles hold them patches them
        // from the dense input)
        if (jbase + ncas == (si.seq_len + kPrefillTileN - 1) / kPrefillTileN)
            append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages,
                            p.Hkv, p.err, si, w.seq, kvh, 0, si.query_len, lane, 32);
    } else if (append) {
        // ------------------- warp 11: this task's share of the cache writes -------------------
        // the G query tiles (one per head of the KV head) on a token tile each write 1/G of its
        // rows; a task does the shares of both its tiles
        for (int b = 0; b < 2; ++b) {
            const int nt = b ? w.ntok1 : w.ntok0, t0 = b ? w.tok1 : w.tok0;
            const int gi = (b ? w.q_head1 : w.q_head) % p.G;
            const int t_begin = t0 + (int)((int64_t)nt * gi / p.G);
            const int t_end = t0 + (int)((int64_t)nt * (gi + 1) / p.G);
            append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages,
                            p.Hkv, p.err, si, w.seq, kvh, t_begin, t_end, lane, 32);
        }
    }
    } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    {
#else
    } else if (warp < 8) {
#endif
        // ------------------------------ softmax (rows) ---------------------------------------
        const int b = warp >> 2;                             // query tile of this warpgroup
        const int r = tid & 127;                             // row = TMEM lane
        const int nb = b ? n1 : n0;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + kColS + b * 128;
        const uint32_t o_addr = tmem + lane_off + kColO + b * D;
        const int row_in_task = (il ? 0 : b) * kPrefillTileM + r;   // interleaved: tile 0's rows
        // this tile's query head and tokens (a cascade task's rows come from its row map)
        const int qh = b ? w.q_head1 : w.q_head;
        const int tok0_b = b ? w.tok1 : w.tok0;
        const int ntok_b = b ? w.ntok1 : w.ntok0;
        const int tok = tok0_b + r;
        // Per KV tile j: its first key kb and the last key this row (lim) and the tile's
        // first row (lim_first) may see. Tiles [0, na) are cache tiles j + jbase with limits
        // (lim_a, lim_first_a); append mode's new tiles j >= na are indexed from the chunk
        // start with limits (lim_b, lim_first_b).
        //   plain: lim_a = prefix + tok (the causal diagonal), all tiles cache tiles;
        //   append: cache tiles show keys [0, prefix) to every row, a new tile's row sees new
        //           keys up to its own token index;
        //   cascade: every shared key (below key_limit) is visible.
        const int na = append ? nc : nmax;
        const int lim_first_b = tok0_b, lim_b = tok;
        const int lim_first_a = cascade || append ? key_limit - 1 : prefix + lim_first_b;
        const int lim_a = cascade || append ? key_limit - 1 : (r < ntok_b ? prefix + tok : 0x7fffffff);
        // FP8 caches: the tiles hold the codes' values, so the K scale of this KV head joins
        // the softmax scale (and the V scale the output, below)
        const float sl2 = p.k_scale ? p.scale_log2 * p.k_scale[kvh] : p.scale_log2;
        float m_ref = -INFINITY, l_sum = 0.f;
        bool alive = true;
        // every break below is taken by the whole warp (tcgen05.ld/st are warp-collective)
        for (int j = 0; j < nb; ++j) {
            if (!__all_sync(0xffffffffu, kSpinOnS ? spin_or_abort(&B.s_full[b], j & 1, p.err, abort_flag)
                                                  : wait_or_abort(&B.s_full[b], j & 1, p.err, abort_flag))) {
                alive = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
            const bool tile_a = j < na;
            const int jj = il ? 2 * j + b : j;                 // this half's j-th KV tile
            const int kb = tile_a ? (jbase + jj) * kPrefillTileN : (j - na) * kPrefillTileN;
            const int lim_j = tile_a ? lim_a : lim_b;
            const int lim_first_j = tile_a ? lim_first_a : lim_first_b;
            // masks as four 32-column words of visible columns, applied by one loop
            uint32_t mw[4];
            bool masked = false;
            if (own) {
                if (kb + kPrefillTileN > prefix) {             // the tile holds new tokens' keys
                    // row r is packed row (token r / G, head r % G): every committed key is
                    // visible, a new token's key only to its tree descendants (causal: to the
                    // tokens from it on). Rows past the unit's take token T - 1's mask (unused).
                    // (Read here, not kept across the loop: no registers taken from it.)
                    const int own_t = min(r / p.G, si.query_len - 1);
                    const bool own_tree = si.mask_kind == PKVA_TREE;
                    const uint64_t own_anc = own_tree ? p.anc[si.anc_off + own_t] : 0ull;
                    masked = true;
                    const int pk = prefix - kb;                // columns below pk: committed keys
#pragma unroll
                    for (int wd = 0; wd < 4; ++wd) {
                        const int lo = 32 * wd;
                        if (own_tree) {                        // committed keys, then the row's ancestors
                            uint32_t m = pk >= lo + 32 ? ~0u : (pk <= lo ? 0u : ((1u << (pk - lo)) - 1u));
                            const int sh = lo - pk;            // bit i of the word is ancestor bit i + sh
                            m |= sh >= 64 ? 0u : sh >= 0 ? (uint32_t)(own_anc >> sh)
                                                         : (sh <= -32 ? 0u : (uint32_t)(own_anc << -sh));
                            mw[wd] = m;
                        } else {                               // causal: columns up to the row's own key
                            const int v = pk + own_t - lo;
                            mw[wd] = v >= 31 ? ~0u : (v < 0 ? 0u : ((2u << v) - 1u));
                        }
                    }
                }
            } else if (kb + kPrefillTileN - 1 > lim_first_j) {        // tile crosses the diagonal
                masked = true;
                const int vis = lim_j - kb;                        // columns <= vis are visible
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
                    const int v = vis - 32 * wd;
                    mw[wd] = v >= 31 ? ~0u : (v < 0 ? 0u : ((2u << v) - 1u));
                }
            }
            if (masked) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (!((mw[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
            }
            // row max as eight independent chains (short dependency depth)
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(sr[i]);
#pragma unroll
            for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(sr[c]));
#pragma unroll
            for (int i = 0; i < 4; ++i) mx8[i] = fmaxf(mx8[i], mx8[i + 4]);
            const float m_tile = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])) * sl2;
            bool need = false;
            float m_new = m_ref;
            if (j == 0) {
                m_ref = m_tile;
            } else {
                need = m_tile > m_ref + kRescaleSlack;
                m_new = fmaxf(m_ref, m_tile);
            }
            const float alpha = need ? exp2f(m_ref - m_new) : 1.f;
            if (need) {
                m_ref = m_new;
                l_sum *= alpha;
            }
            const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
            float ls4[4] = {0.f, 0.f, 0.f, 0.f};
            // P in place: pair c goes to word c (already consumed), then out to S_b[0, 64)
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float x0 = fmaf(__uint_as_float(sr[2 * c]), sl2, -ref);
                const float x1 = fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -ref);
                const float p0 = exp2f(x0);
                const float p1 = exp2f(x1);
                ls4[c & 3] += p0 + p1;
                sr[c] = pack_bf16x2(p0, p1);
            }
            l_sum += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
            tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            if (__any_sync(0xffffffffu, need)) {
                // rescale O_b (done with S, so its registers are free). O_b is complete for
                // tile j-1: S_b of tile j was committed after that PV was issued.
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(o_addr + c * 32, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    tmem_st32(o_addr + c * 32, ov);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&B.p_full[b]);
        }
        // ---- epilogue (cascade): unnormalised O, max and sum -> the row's split slot --------
        if (cascade) {
            // where this row's partial goes (slot * 16 + row in unit), or -1
            const int part_idx = p.crowmap[(int64_t)ci * 2 * kPrefillTileM + row_in_task];
            const bool real_row = part_idx >= 0;
            if (il) {
                // combine the halves: each warpgroup hands its (max, sum) over through Q tile
                // 1's shared memory (never loaded in this mode), then writes half the columns
                float* xch = reinterpret_cast<float*>(sm + L::kOffQ + L::kTileBytes);    // [2][128][2]
                const bool mine = nb > 0 && alive;
                xch[(b * kPrefillTileM + r) * 2] = mine ? m_ref : -INFINITY;
                xch[(b * kPrefillTileM + r) * 2 + 1] = mine ? l_sum : 0.f;
                asm volatile("bar.sync 1, 256;" ::: "memory");
                const float m0 = xch[r * 2], l0 = xch[r * 2 + 1];
                const float m1 = xch[(kPrefillTileM + r) * 2], l1 = xch[(kPrefillTileM + r) * 2 + 1];
                const float M = fmaxf(m0, m1);
                const float w0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
                const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
                const bool waited = __all_sync(0xffffffffu, alive && !*abort_flag &&
                                                                (n0 == 0 || wait_or_abort(&B.o_ready[0], 0, p.err, abort_flag)) &&
                                                                (n1 == 0 || wait_or_abort(&B.o_ready[1], 0, p.err, abort_flag)));
                if (waited && cw.own != 2) {
                    tc_fence_after();
                    float* dst = p.part_o + (int64_t)(part_idx < 0 ? 0 : part_idx) * D;
                    const float vsc = p.v_scale ? p.v_scale[kvh] : 1.f;
                    const float f0 = w0 * vsc, f1 = w1 * vsc;
                    const uint32_t o0 = tmem + lane_off + kColO, o1 = o0 + D;
#pragma unroll
                    for (int c = b * (D / 64); c < (b + 1) * (D / 64); ++c) {
                        uint32_t v0[32], v1[32];
                        if (n0 > 0) tmem_ld32(o0 + c * 32, v0);
                        if (n1 > 0) tmem_ld32(o1 + c * 32, v1);
                        tmem_wait_ld();
                        if (real_row) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                float4 v;
                                v.x = (n0 > 0 ? __uint_as_float(v0[e]) * f0 : 0.f) + (n1 > 0 ? __uint_as_float(v1[e]) * f1 : 0.f);
                                v.y = (n0 > 0 ? __uint_as_float(v0[e + 1]) * f0 : 0.f) +
                                      (n1 > 0 ? __uint_as_float(v1[e + 1]) * f1 : 0.f);
                                v.z = (n0 > 0 ? __uint_as_float(v0[e + 2]) * f0 : 0.f) +
                                      (n1 > 0 ? __uint_as_float(v1[e + 2]) * f1 : 0.f);
                                v.w = (n0 > 0 ? __uint_as_float(v0[e + 3]) * f0 : 0.f) +
                                      (n1 > 0 ? __uint_as_float(v1[e + 3]) * f1 : 0.f);
                                *reinterpret_cast<float4*>(dst + c * 32 + e) = v;
                            }
                        }
                    }
                    if (real_row && b == 0)
                        *reinterpret_cast<float2*>(p.part_ml + (int64_t)part_idx * 2) = make_float2(M, l0 * w0 + l1 * w1);
                }
                if (waited && cw.own == 2) {
                    // one task over all of the sequence's keys: O / l straight to the row
                    tc_fence_after();
                    const bool real = r < cw.ntok * p.G;
                    const float Lr = l0 * w0 + l1 * w1;
                    const float inv = (Lr > 0.f ? 1.f / Lr : 0.f) * (p.v_scale ? p.v_scale[kvh] : 1.f);
                    const float f0 = w0 * inv, f1 = w1 * inv;
                    __nv_bfloat16* dst = p.out + ((int64_t)(si.q_start + r / p.G) * p.Hq + kvh * p.G + r % p.G) * D;
                    const uint32_t o0 = tmem + lane_off + kColO, o1 = o0 + D;
#pragma unroll
                    for (int c = b * (D / 64); c < (b + 1) * (D / 64); ++c) {
                        uint32_t v0[32], v1[32];
                        if (n0 > 0) tmem_ld32(o0 + c * 32, v0);
                        if (n1 > 0) tmem_ld32(o1 + c * 32, v1);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            float x[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                x[q] = (n0 > 0 ? __uint_as_float(v0[e + q]) * f0 : 0.f) +
                                       (n1 > 0 ? __uint_as_float(v1[e + q]) * f1 : 0.f);
                            if (real)
                                *reinterpret_cast<uint4*>(dst + c * 32 + e) =
                                    make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                               pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
                        }
                    }
                }
            } else if (nb > 0 && alive && __all_sync(0xffffffffu, wait_or_abort(&B.o_ready[b], 0, p.err, abort_flag))) {
                tc_fence_after();
                float* dst = p.part_o + (int64_t)(part_idx < 0 ? 0 : part_idx) * D;
                // FP8 caches: the V scale of this KV head, as on every other partial
                const float vsc = p.v_scale ? p.v_scale[kvh] : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(o_addr + c * 32, ov);
                    tmem_wait_ld();
                    if (real_row) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(dst + c * 32 + e) =
                                make_float4(__uint_as_float(ov[e]) * vsc, __uint_as_float(ov[e + 1]) * vsc,
                                            __uint_as_float(ov[e + 2]) * vsc, __uint_as_float(ov[e + 3]) * vsc);
                    }
                }
                if (real_row)
                    *reinterpret_cast<float2*>(p.part_ml + (int64_t)part_idx * 2) = make_float2(m_ref, l_sum);
            }
            // all 256 softmax threads: count one arrival per unit touched, then merge the
            // units this task completed. Every MMA has finished here (both warpgroups waited
            // for their tiles' last PV), so the Q tiles' shared memory is free for the flags.
            __threadfence();
            asm volatile("bar.sync 1, 256;" ::: "memory");
            int* cnt = reinterpret_cast<int*>(sm + L::kOffQ);      // [256] rows of each completed unit, else 0
            int* uid = cnt + 256;                                // [256]
            int* pref = uid + 256;                               // [256] compacted prefix sums
            int* cuid = pref + 256;                              // [256] compacted unit ids
            const bool aborted = *abort_flag != 0;
            for (int i = tid; i < cw.unit_cnt; i += 256) {
                const int u = p.cunits[cw.unit_off + i];
                const bool done = !aborted && atomicAdd(&p.counters[u], 1) == p.units[u].arrivals - 1;
                if (done) p.counters[u] = 0;        // every arrival is in: ready for the next run
                cnt[i] = done ? p.units[u].row_count : 0;
                uid[i] = u;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            int* totals = cuid + 256;                            // [2]: rows, units
            if (tid == 0) {                          // compact the completed units (a few hundred at most)
                int n = 0, rows = 0;
                for (int i = 0; i < cw.unit_cnt; ++i)
                    if (cnt[i]) {
                        pref[n] = rows;
                        cuid[n++] = uid[i];
                        rows += cnt[i];
                    }
                totals[0] = rows;
                totals[1] = n;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            __threadfence();
            const int total = totals[0], n_done = totals[1];
            if (n_done > 0)
                merge_units<D>(warp, 8, lane, cuid, pref, n_done, total, p.units, p.part_o, p.part_ml, p.seqs,
                                p.out, p.Hq, p.G);
        }
        // ---- epilogue: O / l -> bf16 rows --------------------------------------------------
        else if (nb > 0 && alive && __all_sync(0xffffffffu, wait_or_abort(&B.o_ready[b], 0, p.err, abort_flag))) {
            tc_fence_after();
            const bool real_row = r < ntok_b;
            float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            if (p.v_scale) inv *= p.v_scale[kvh];
            __nv_bfloat16* dst = p.out + ((int64_t)(si.q_start + tok) * p.Hq + qh) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld32(o_addr + c * 32, ov);
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
#if PKVA_PREFILL_RS
    }
    }
#else
    } else if (own && p.append && warp == kPThreads / 32) {
        // ------------------- warp 11: a tensor-core verify task's cache writes ----------------
        // the task with the unit's last KV tiles writes the sequence's new rows of its KV head
        // (no other task reads those cache slots: any task whose tiles hold them patches them
        // from the dense input)
        if (jbase + ncas == (si.seq_len + kPrefillTileN - 1) / kPrefillTileN)
            append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages,
                            p.Hkv, p.err, si, w.seq, kvh, 0, si.query_len, lane, 32);
    } else if (append) {
        // ------------------- warp 11: this task's share of the cache writes -------------------
        // the G query tiles (one per head of the KV head) on a token tile each write 1/G of its
        // rows; a task does the shares of both its tiles
        for (int b = 0; b < 2; ++b) {
            const int nt = b ? w.ntok1 : w.ntok0, t0 = b ? w.tok1 : w.tok0;
            const int gi = (b ? w.q_head1 : w.q_head) % p.G;
            const int t_begin = t0 + (int)((int64_t)nt * gi / p.G);
            const int t_end = t0 + (int)((int64_t)nt * (gi + 1) / p.G);
            append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages,
                            p.Hkv, p.err, si, w.seq, kvh, t_begin, t_end, lane, 32);
        }
    }
#endif
    // all roles done (the MMA thread waited for its last MMA): TMEM and shared memory are
    // free for the block's next task
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        uint64_t* b = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
        for (int i = 0; i < kNumBars; ++i) mbar_inval(&b[i]);
    }
}

