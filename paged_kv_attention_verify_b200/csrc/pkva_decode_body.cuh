// Decode / verify task bodies (K-D), shared by the stand-alone decode kernels and the
// unified attention kernel. See pkva_decode.cu for the design notes.
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
namespace dec {

// The threads that run one decode task: a whole block, or one half of a larger block
// (each half with its own shared memory and named barrier).
struct Group {
    int tid;        // thread index within the group
    int n;          // threads in the group (a multiple of 32)
    int bar;        // named barrier id
    __device__ __forceinline__ void sync() const {
        asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(n) : "memory");
    }
};


constexpr int kBoxBytes = kPageSize * 128;     // one TMA box: 16 rows x 64 bf16
constexpr int kBtSlice = kDecodeMaxPages;      // block-table entries staged per task
constexpr float kRescaleSlack = 8.f;           // log2 units a stale row max may lag (mma body)

constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory map of one task. NR = rows the launch is compiled for; QF = whether the
// CUDA-core body's staged Q and P buffers are present; NW = page-streaming warps; NS =
// stages per warp; EB = bytes per cached K/V element (2 bf16, 1 FP8).
template <int D, int NR, bool QF, int NW, int NS_, int EB = 2>
struct DecodeCfg {
    static constexpr int NS = NS_;
    static constexpr int PAGE_BYTES = kPageSize * D * EB;
    static constexpr int STAGE_BYTES = 2 * PAGE_BYTES;              // K page + V page
    static constexpr int HALF = D / 2;                              // columns per lane half
    static constexpr int QROW = D + 8;                              // floats per staged Q row
    static constexpr int OPL = D / 32;                              // output columns per lane
    static constexpr int RING = NW * NS * STAGE_BYTES;
    static constexpr int OFF_Q = RING;
    static constexpr int OFF_P = OFF_Q + (QF ? NR * QROW * 4 : 0);
    static constexpr int OFF_BT = OFF_P + (QF ? NW * kPageSize * NR * 4 : 0);
    static constexpr int OFF_LIM = OFF_BT + kBtSlice * 4;
    static constexpr int OFF_ANC = align_up(OFF_LIM + NR * 4, 8);
    static constexpr int OFF_OUT = OFF_ANC + NR * 8;
    static constexpr int OFF_BAR = align_up(OFF_OUT + NR * 4, 8);
    static constexpr int OFF_FLAG = OFF_BAR + NW * NS * 8;
    // tensor-core body with two n-tiles: Q rows staged in shared memory (swizzled 16-byte
    // chunks) and read per page with ldmatrix, instead of 32 registers held through the loop
    static constexpr bool QB = !QF && NR > 8;
    static constexpr int OFF_QB = align_up(OFF_FLAG + 16, 128);
    static constexpr int BYTES = QB ? OFF_QB + NR * D * 2 : OFF_FLAG + 16;
    static constexpr int ALLOC = BYTES + 1008;                     // room to align to 1024
    static_assert(NW * NR * (D + 2) * 4 <= RING, "combine buffers must fit in the ring");
    static_assert(D == 64 || D == 128, "head_dim");
};

__device__ __forceinline__ int q_row_index(const DecodeParams& p, const SeqInfo& si, const DecodeWork& w,
                                           int r) {
    const int rr = w.row_begin + r;
    const int t = rr / p.G;
    const int g = rr - t * p.G;
    return (si.q_start + t) * p.Hq + w.kv_head * p.G + g;
}

// Per-task set-up shared by both bodies: barriers (unless the warps set up their own),
// block-table slice, row records.
template <int NR, int NS, int NW>
__device__ __forceinline__ void task_setup(const Group& grp, const DecodeParams& p, const DecodeWork& w,
                                           const SeqInfo& si,
                                           int* bts, int* rlim, uint64_t* ranc, int* rout, uint64_t* bars,
                                           int* flag, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                           bool init_bars = true) {
    const int tid = grp.tid;
    const int R = w.row_count;
    const int npg = w.page_end - w.page_begin;
    const int prefix = si.seq_len - si.query_len;
    if (tid == 0) {
        if (init_bars) {
            for (int i = 0; i < NW * NS; ++i) mbar_init(&bars[i], 1);
            fence_mbar_init();
            prefetch_tensormap(tmK);
            prefetch_tensormap(tmV);
        }
        flag[0] = 0;
        flag[1] = 0;
    }
    // block-table slice of this task; an entry out of range is flagged and its page is
    // loaded from a fully out-of-bounds box, which TMA fills with zeros
    const int32_t* btrow = p.block_table + (int64_t)w.seq * p.bt_stride + w.page_begin;
    for (int i = tid; i < npg; i += grp.n) {
        const int ph = btrow[i];
        const bool bad = ph < 0 || ph >= p.num_pages;
        if (bad) atomicOr(p.err, PKVA_DEVERR_BAD_PAGE);
        bts[i] = bad ? -1 : ph;
    }
    // per-row records: output row, causal limit, tree ancestor mask
    if (tid < NR) {
        const int r = tid;
        if (r < R) {
            const int t = (w.row_begin + r) / p.G;
            rout[r] = q_row_index(p, si, w, r);
            if (si.mask_kind == PKVA_CAUSAL) {
                rlim[r] = prefix + t;
                ranc[r] = 0ull;
            } else {
                rlim[r] = prefix - 1;
                ranc[r] = p.anc[si.anc_off + t];
            }
        } else {
            rout[r] = -1;
            rlim[r] = 0x7fffffff;
            ranc[r] = 0ull;
        }
    }
}

// Load page #i of this warp's stream (lane 0 only); ph is its physical page, -1 for none.
// bf16: K and V as 16 x 64 boxes (128-byte swizzle). FP8: the K page as one 16 x D-byte box
// (128- or 64-byte swizzle) and the transposed V page as one box of D/8 rows of 128 bytes.
template <int D, int NS, int STAGE_BYTES, int PAGE_BYTES, bool FP8 = false>
__device__ __forceinline__ void issue_page_at(const DecodeParams& p, const DecodeWork& w, int ph, uint8_t* ring,
                                              uint64_t* bar, int i, const CUtensorMap* tmK, const CUtensorMap* tmV) {
    const int stage = i % NS;
    const int blk = ph >= 0 ? ph * p.Hkv + w.kv_head : -1;       // (page, KV head) block; -1 reads zeros
    uint8_t* dst = ring + stage * STAGE_BYTES;
    mbar_arrive_expect_tx(&bar[stage], STAGE_BYTES);
    if constexpr (FP8) {
        tma_load_2d(dst, tmK, &bar[stage], 0, blk * kPageSize);
        tma_load_2d(dst + PAGE_BYTES, tmV, &bar[stage], 0, blk * (D / 8));
    } else {
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {
            tma_load_2d(dst + b * kBoxBytes, tmK, &bar[stage], b * 64, blk * kPageSize);
            tma_load_2d(dst + PAGE_BYTES + b * kBoxBytes, tmV, &bar[stage], b * 64, blk * kPageSize);
        }
    }
}

// Load page #i of this warp's stream from the staged block-table slice (lane 0 only).
template <int D, int NS, int STAGE_BYTES, int PAGE_BYTES, int NW, bool FP8 = false>
__device__ __forceinline__ void issue_page(const DecodeParams& p, const DecodeWork& w, const int* bts,
                                           uint8_t* ring, uint64_t* bar, int warp, int i,
                                           const CUtensorMap* tmK, const CUtensorMap* tmV) {
    issue_page_at<D, NS, STAGE_BYTES, PAGE_BYTES, FP8>(p, w, bts[warp + NW * i], ring, bar, i, tmK, tmV);
}

// FP8 page body: the M row m of the K operand (and of S^T) holds key sigma(m) of the page,
// so that after the in-register transpose of P its k slots line up with the keys the
// transposed V operand delivers (four consecutive keys per lane, see decode_mma_task).
__device__ __forceinline__ int fp8_key_of_row(int m) { return ((m & 7) >> 1) * 4 + (m >> 3) * 2 + (m & 1); }

// One bf16 page (16 keys) for the rows one warp holds (NT n-tiles of 8 rows): S^T = K Q^T,
// the row masks, the lazily rescaled online softmax and O^T += V^T P^T. Ks / Vs: the page's
// K and V (16 x 64 boxes, 128-byte swizzle); Q from qs (rows staged in shared memory, 16-byte
// chunk c of row r at c ^ (r & 7)) when QB, else from the fragments in qf. Slots past the
// sequence's end hold stale cache data: their V rows are zeroed in shared memory first
// (every warp that reads the page writes the same zeros, so several may share it).
template <int D, int NT, bool QB>
__device__ __forceinline__ void bf16_page(const uint8_t* Ks, uint8_t* Vs, const uint8_t* qs,
                                          const uint32_t (&qf)[NT][QB ? 1 : D / 16][2], int kbase, int prefix,
                                          int seq_len, int min_lim, const int (&lim)[NT][2],
                                          const uint64_t (&anc)[NT][2], float sl2, float (&o)[D / 16][NT][4],
                                          float (&mref)[NT][2], float (&lsum)[NT][2]) {
    constexpr int KS = D / 16;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int mi = lane >> 3, mr = lane & 7;
    const int k_key = mr + (mi & 1) * 8, k_chunk = mi >> 1;          // K: A operand, keys on M
    const int v_key = mr + (mi >> 1) * 8, v_chunk = mi & 1;          // V: A operand of V^T (trans)
    // -- S^T = K Q^T (16 keys x 8 rows per n-tile) ------------------------------------
    // even and odd k-steps accumulate into separate tiles (two dependent MMA chains of half
    // the length), added at the end
    float s[NT][4], s2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
    if constexpr (QB) {
#pragma unroll
        for (int k2 = 0; k2 < KS; k2 += 2) {
            uint32_t qb[NT][4];              // b fragments of k-steps k2 and k2 + 1
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int qr = nt * 8 + (lane & 7), qc = 2 * k2 + (lane >> 3);
                ldmatrix_x4(qb[nt], qs + qr * (D * 2) + ((qc ^ (qr & 7)) << 4));
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int cg = (k2 + kk) * 2 + k_chunk;
                uint32_t a[4];
                ldmatrix_x4(a, Ks + (cg >> 3) * kBoxBytes + k_key * 128 + (((cg & 7) ^ (k_key & 7)) << 4));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(kk ? s2[nt] : s[nt], a, &qb[nt][2 * kk]);
            }
        }
    } else {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int cg = ks * 2 + k_chunk;
            uint32_t a[4];
            ldmatrix_x4(a, Ks + (cg >> 3) * kBoxBytes + k_key * 128 + (((cg & 7) ^ (k_key & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816((ks & 1) ? s2[nt] : s[nt], a, qf[nt][ks]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];

    // -- mask ---------------------------------------------------------------------------
    const bool page_all = (kbase + kPageSize - 1) <= min_lim;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kpos = kbase + g + 8 * h;
                float v = s[nt][2 * h + e] * sl2;
                if (!page_all) {
                    bool allow = kpos <= lim[nt][e];
                    if (!allow && kpos >= prefix && kpos < seq_len)
                        allow = (anc[nt][e] >> (kpos - prefix)) & 1ull;
                    v = allow ? v : -INFINITY;
                }
                s[nt][2 * h + e] = v;
            }
    // -- lazy rescale: only when some score passed its row's reference by the slack (or the
    //    row has no reference yet). Each lane checks its own scores; the row max over the
    //    page (shuffles across the lanes of a column) is taken only in that rare case.
    bool need = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float mx = fmaxf(s[nt][e], s[nt][2 + e]);
            need |= mx > mref[nt][e] + kRescaleSlack || (mref[nt][e] == -INFINITY && mx != -INFINITY);
        }
    if (__any_sync(0xffffffffu, need)) {
        float cmax[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = fmaxf(s[nt][e], s[nt][2 + e]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                cmax[nt][e] = mx;
            }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float mnew = fmaxf(mref[nt][e], cmax[nt][e]);
                if (mnew != mref[nt][e]) {
                    const float alpha = mref[nt][e] == -INFINITY ? 0.f : exp2f(mref[nt][e] - mnew);
                    mref[nt][e] = mnew;
                    lsum[nt][e] *= alpha;
#pragma unroll
                    for (int dt = 0; dt < KS; ++dt) {
                        o[dt][nt][e] *= alpha;
                        o[dt][nt][2 + e] *= alpha;
                    }
                }
            }
    }
    // -- P = exp2(S - ref), row sums, P^T as the B operand (transpose in registers) -----
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float ref = mref[nt][e] == -INFINITY ? 0.f : mref[nt][e];
            pv[e] = exp2f(s[nt][e] - ref);
            pv[2 + e] = exp2f(s[nt][2 + e] - ref);
            lsum[nt][e] += pv[e] + pv[2 + e];
        }
        pb[nt][0] = movmatrix_trans(pack_bf16x2(pv[0], pv[1]));   // keys 0..7
        pb[nt][1] = movmatrix_trans(pack_bf16x2(pv[2], pv[3]));   // keys 8..15
    }
    // slots past the sequence's end hold stale cache data: zero those V rows so that
    // P = 0 times a non-finite value cannot reach the accumulators
    const int nvalid = seq_len - kbase;
    if (nvalid < kPageSize) {
        for (int idx = lane; idx < (kPageSize - nvalid) * (D / 8); idx += 32) {
            const int row = nvalid + idx / (D / 8);
            const int cg = idx % (D / 8);
            *reinterpret_cast<uint4*>(Vs + (cg >> 3) * kBoxBytes + row * 128 + (cg & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
    }
    // -- O^T += V^T P^T -----------------------------------------------------------------
    {
#pragma unroll
        for (int dt = 0; dt < KS; ++dt) {
            const int cg = dt * 2 + v_chunk;
            uint32_t a[4];
            ldmatrix_x4_trans(a, Vs + (cg >> 3) * kBoxBytes + v_key * 128 + (((cg & 7) ^ (v_key & 7)) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[dt][nt], a, pb[nt]);
        }
    }
}

// Merge the four warps' (max, sum, unnormalised output) held in cm/cl/co, then either
// write the rows (whole unit) or a split partial; the last split of a unit merges all
// partials. Every thread of the CTA calls this.
template <int D, int NR, int NW>
__device__ __forceinline__ void merge_and_store(const Group& grp, const DecodeParams& p, const DecodeWork& w,
                                                const float* cm, const float* cl, const float* co,
                                                const int* rout, int* flag) {
    const int tid = grp.tid;
    const int R = w.row_count;
    const bool split = w.unit >= 0;
    int slot = 0;
    if (split) slot = p.units[w.unit].slot_base + w.split;
    for (int idx = tid; idx < R * (D / 2); idx += grp.n) {
        const int r = idx / (D / 2);
        const int c = (idx - r * (D / 2)) * 2;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) M = fmaxf(M, cm[ww * NR + r]);
        float o0 = 0.f, o1 = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int ww = 0; ww < NW; ++ww) {
                const float f = exp2f(cm[ww * NR + r] - M);
                const float2 v = *reinterpret_cast<const float2*>(co + (ww * NR + r) * D + c);
                o0 = fmaf(f, v.x, o0);
                o1 = fmaf(f, v.y, o1);
                L = fmaf(f, cl[ww * NR + r], L);
            }
        }
        if (!split) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            *reinterpret_cast<__nv_bfloat162*>(p.out + (int64_t)rout[r] * D + c) =
                __floats2bfloat162_rn(o0 * inv, o1 * inv);
        } else {
            *reinterpret_cast<float2*>(p.part_o + ((int64_t)slot * kDecodeRowsMax + r) * D + c) =
                make_float2(o0, o1);
            if (c == 0)
                *reinterpret_cast<float2*>(p.part_ml + ((int64_t)slot * kDecodeRowsMax + r) * 2) =
                    make_float2(M, L);
        }
    }
    if (!split) return;

    // ---- split-KV combine: the last task of the unit to finish merges all partials -------
    __threadfence();
    grp.sync();
    if (tid == 0) {
        const int prev = atomicAdd(&p.counters[w.unit], 1);
        flag[0] = (prev == p.units[w.unit].arrivals - 1);
        if (flag[0]) p.counters[w.unit] = 0;        // every arrival is in: ready for the next run
    }
    grp.sync();
    if (!flag[0]) return;
    __threadfence();
    const int32_t uid = w.unit;
    const int pref0 = 0;
    merge_units<D>(tid >> 5, grp.n >> 5, tid & 31, &uid, &pref0, 1, w.row_count, p.units, p.part_o, p.part_ml,
                   p.seqs, p.out, p.Hq, p.G);
}

// =====================================================================================
// Tensor-core page body (mma.sync): keys on M, the group's rows on N.
// =====================================================================================
// One decode/verify task on the tensor-core page body. Every thread of the block calls it;
// warps [0, NW) stream pages, any further warps only take part in the block barriers.
//
// FP8 (E4M3 codes, one scale per KV head): the same tiles in f16 (every E4M3 value is an
// f16 value, and bf16 Q converts exactly in f16's normal range). ldmatrix reads the codes
// as 16-bit pairs, so a lane holds four consecutive bytes of a row where the bf16 layout
// would give it two pairs eight apart; the k slots of both operands are permuted alike:
//   QK^T: k slots (2t, 2t+1) and (2t+8, 2t+9) of a 16-column step take head-dim columns
//         (4t, 4t+1) and (4t+2, 4t+3); Q is loaded (or staged) in that order;
//   PV:   V is cached transposed per page ([D][16] bytes), so its rows are head-dim
//         columns and a lane holds keys 4t..4t+3; S^T's M rows are permuted
//         (fp8_key_of_row) so that after the transpose of P its k slots (2t, 2t+1) and
//         (2t+8, 2t+9) are exactly keys (4t, 4t+1) and (4t+2, 4t+3).
// The K scale folds into the softmax scale and the V scale into the output.
template <int D, int NT, int NW, int NS, bool FP8 = false>
__device__ __forceinline__ void decode_mma_task(const Group& grp, const DecodeParams& p, int task,
                                                const CUtensorMap& tmK, const CUtensorMap& tmV, uint8_t* sm) {
    constexpr int NR = NT * 8;
    using C = DecodeCfg<D, NR, false, NW, NS, FP8 ? 1 : 2>;
    constexpr int KS = D / 16;                    // k-steps of QK^T; d-tiles of PV

    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;       // fragment row group / thread-in-group
    const DecodeWork w = p.work[task];
    const SeqInfo si = p.seqs[w.seq];

    int* bts = reinterpret_cast<int*>(sm + C::OFF_BT);
    int* rlim = reinterpret_cast<int*>(sm + C::OFF_LIM);
    uint64_t* ranc = reinterpret_cast<uint64_t*>(sm + C::OFF_ANC);
    int* rout = reinterpret_cast<int*>(sm + C::OFF_OUT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    int* flag = reinterpret_cast<int*>(sm + C::OFF_FLAG);

    const int R = w.row_count;
    const int npg = w.page_end - w.page_begin;
    const int prefix = si.seq_len - si.query_len;
    const int n_my = (warp < NW && npg > warp) ? (npg - warp + NW - 1) / NW : 0;
    uint8_t* ring = sm + warp * C::NS * C::STAGE_BYTES;    // used only by warps < NW
    uint64_t* bar = bars + warp * C::NS;

    // each streaming warp sets up its own stages and starts its first pages at once,
    // reading their block-table entries directly; the rest of the set-up overlaps them
    if (warp < NW && lane == 0) {
        for (int i = 0; i < C::NS; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
        fence_proxy_async_smem();                  // the previous task's generic accesses come first
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        const int32_t* btrow = p.block_table + (int64_t)w.seq * p.bt_stride + w.page_begin;
        for (int i = 0; i < C::NS && i < n_my; ++i) {
            int ph = btrow[warp + NW * i];
            if (ph < 0 || ph >= p.num_pages) ph = -1;     // flagged by the slice staging below
            issue_page_at<D, C::NS, C::STAGE_BYTES, C::PAGE_BYTES, FP8>(p, w, ph, ring, bar, i, &tmK, &tmV);
        }
    }
    task_setup<NR, C::NS, NW>(grp, p, w, si, bts, rlim, ranc, rout, bars, flag, &tmK, &tmV, false);

    // Q^T as the B operand: row (column of S^T) nt*8+g, k = d. One n-tile: pairs straight
    // from global into registers. Two: rows staged in shared memory, chunk c of row r at
    // chunk c ^ (r & 7), read per page with ldmatrix (keeps the page loop out of spilling).
    constexpr int QREG = C::QB ? 1 : KS;
    uint32_t qf[NT][QREG][2];
    uint8_t* qs = sm + C::OFF_QB;
    if constexpr (C::QB && FP8) {
        // f16, each 16-column group stored as columns 0,1,4,5,8,9,12,13, 2,3,6,7,10,11,14,15
        for (int idx = tid; idx < NR * (D / 16); idx += grp.n) {
            const int r = idx / (D / 16), j = idx - r * (D / 16);
            uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi[4] = {0u, 0u, 0u, 0u};
            if (r < R) {
                const uint4* src = reinterpret_cast<const uint4*>(p.q + (int64_t)q_row_index(p, si, w, r) * D + j * 16);
                const uint4 a = src[0], b = src[1];
                const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};   // bf16 pairs (2t', 2t'+1)
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    float x0, x1, x2, x3;
                    bf16x2_to_f32(wv[2 * t], x0, x1);
                    bf16x2_to_f32(wv[2 * t + 1], x2, x3);
                    lo[t] = pack_f16x2(x0, x1);          // columns 4t, 4t+1
                    hi[t] = pack_f16x2(x2, x3);          // columns 4t+2, 4t+3
                }
            }
            *reinterpret_cast<uint4*>(qs + r * (D * 2) + (((2 * j) ^ (r & 7)) << 4)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            *reinterpret_cast<uint4*>(qs + r * (D * 2) + (((2 * j + 1) ^ (r & 7)) << 4)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        }
    } else if constexpr (C::QB) {
        for (int idx = tid; idx < NR * (D / 8); idx += grp.n) {
            const int r = idx / (D / 8), c = idx - r * (D / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < R) v = *reinterpret_cast<const uint4*>(p.q + (int64_t)q_row_index(p, si, w, r) * D + c * 8);
            *reinterpret_cast<uint4*>(qs + r * (D * 2) + ((c ^ (r & 7)) << 4)) = v;
        }
    } else if constexpr (FP8) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r = nt * 8 + g;
            if (r < R) {
                const __nv_bfloat16* qp = p.q + (int64_t)q_row_index(p, si, w, r) * D + 4 * t4;
#pragma unroll
                for (int ks = 0; ks < QREG; ++ks) {
                    const uint2 v = *reinterpret_cast<const uint2*>(qp + ks * 16);
                    float x0, x1, x2, x3;
                    bf16x2_to_f32(v.x, x0, x1);
                    bf16x2_to_f32(v.y, x2, x3);
                    qf[nt][ks][0] = pack_f16x2(x0, x1);
                    qf[nt][ks][1] = pack_f16x2(x2, x3);
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < QREG; ++ks) qf[nt][ks][0] = qf[nt][ks][1] = 0u;
            }
        }
    } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int r = nt * 8 + g;
            if (r < R) {
                const __nv_bfloat16* qp = p.q + (int64_t)q_row_index(p, si, w, r) * D + 2 * t4;
#pragma unroll
                for (int ks = 0; ks < QREG; ++ks) {
                    qf[nt][ks][0] = *reinterpret_cast<const uint32_t*>(qp + ks * 16);
                    qf[nt][ks][1] = *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8);
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < QREG; ++ks) qf[nt][ks][0] = qf[nt][ks][1] = 0u;
            }
        }
    }
    grp.sync();

    // this thread's columns: c = nt*8 + 2*t4 + e
    int lim[NT][2];
    uint64_t anc[NT][2];
    int min_lim = 0x7fffffff;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = nt * 8 + 2 * t4 + e;
            lim[nt][e] = rlim[c];
            anc[nt][e] = ranc[c];
        }
    for (int r = 0; r < R; ++r) min_lim = min(min_lim, rlim[r]);

    float o[KS][NT][4];           // O^T tiles: [d-tile][n-tile]{(d g, c), (d g, c+1), (d g+8, c), (d g+8, c+1)}
    float mref[NT][2], lsum[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            mref[nt][e] = -INFINITY;
            lsum[nt][e] = 0.f;
        }
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[dt][nt][i] = 0.f;
    }

    // ldmatrix row addresses: matrix mi = lane >> 3 supplies its rows from lanes 8mi..8mi+7
    const int mi = lane >> 3, mr = lane & 7;
    const int k_key = mr + (mi & 1) * 8, k_chunk = mi >> 1;          // K: A operand, keys on M
    const int v_key = mr + (mi >> 1) * 8, v_chunk = mi & 1;          // V: A operand of V^T (trans)
    const int k8_key = fp8_key_of_row(mr + 8 * (mi & 1)), k8_chunk = mi >> 1;   // FP8 K rows
    const int v8_row = 8 * (mi & 1) + mr + 16 * (mi >> 1);           // FP8 V^T: head-dim row in a pair of d-tiles
    const float sl2 = FP8 ? p.scale_log2 * p.k_scale[w.kv_head] : p.scale_log2;
    bool ok = true;
    int waited = 0;

    if constexpr (FP8) {
        // FP8 pages are half the bytes of bf16 ones, so a warp takes two pages (two stages) per
        // iteration: their tiles are independent until the shared max, which halves the
        // dependent chains per byte.
        for (int i = 0; i < n_my; i += 2) {
            const bool two = i + 1 < n_my;               // the pair's second page exists
            bool got = mbar_wait_bounded(&bar[i % C::NS], (i / C::NS) & 1, p.err, PKVA_DEVERR_TIMEOUT);
            if (two && got) got = mbar_wait_bounded(&bar[(i + 1) % C::NS], ((i + 1) / C::NS) & 1, p.err,
                                                    PKVA_DEVERR_TIMEOUT);
            waited = i + (two ? 2 : 1);
            if (__any_sync(0xffffffffu, !got)) {
                ok = false;
                break;
            }
            int kbase[2];
            uint8_t* Kp[2];
            uint8_t* Vp[2];
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                kbase[pp] = (w.page_begin + warp + NW * (i + pp)) * kPageSize;
                Kp[pp] = ring + ((i + pp) % C::NS) * C::STAGE_BYTES;
                Vp[pp] = Kp[pp] + C::PAGE_BYTES;
            }
            if (p.append) {
                // fused append: the new tokens' rows are the dense input's codes, not the cache's
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    if (pp == 1 && !two) break;
                    if (kbase[pp] + kPageSize > prefix && kbase[pp] < si.seq_len) {
                        const int r0 = max(prefix - kbase[pp], 0), r1 = min(si.seq_len - kbase[pp], kPageSize);
                        patch_page_rows_fp8<D>(Kp[pp], Vp[pp], p.k_new, p.v_new, si, p.Hkv, w.kv_head, r0, r1,
                                               kbase[pp] + r0 - prefix, lane, p.k_scale[w.kv_head],
                                               p.v_scale[w.kv_head]);
                    }
                }
                __syncwarp();
            }
            // -- S^T = K Q^T for both pages ------------------------------------------------
            float s[2][NT][4];
#pragma unroll
            for (int pp = 0; pp < 2; ++pp)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[pp][nt][e] = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KS; k2 += 2) {
                uint32_t qb[NT][4];                      // b fragments of k-steps k2 and k2 + 1
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if constexpr (C::QB) {
                        const int qr = nt * 8 + (lane & 7), qc = 2 * k2 + (lane >> 3);
                        ldmatrix_x4(qb[nt], qs + qr * (D * 2) + ((qc ^ (qr & 7)) << 4));
                    } else {
                        qb[nt][0] = qf[nt][k2][0];
                        qb[nt][1] = qf[nt][k2][1];
                        qb[nt][2] = qf[nt][k2 + 1][0];
                        qb[nt][3] = qf[nt][k2 + 1][1];
                    }
                }
                // codes of keys sigma(g), sigma(g+8), head-dim bytes [16 k, 16 k + 16) for
                // k = k2, k2 + 1 (K page: rows of D bytes, 128- or 64-byte swizzle)
                const int kc = k2 + k8_chunk;
                const int sw = D == 128 ? (kc ^ (k8_key & 7)) : (kc ^ ((k8_key >> 1) & 3));
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    if (pp == 1 && !two) break;
                    uint32_t r[4];
                    ldmatrix_x4(r, Kp[pp] + k8_key * D + (sw << 4));
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        uint32_t a[4];
                        e4m3x4_to_f16x2x2(r[2 * kk], a[0], a[2]);
                        e4m3x4_to_f16x2x2(r[2 * kk + 1], a[1], a[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_f16_16816(s[pp][nt], a, &qb[nt][2 * kk]);
                    }
                }
            }
            // -- mask; this lane's max of each row over the pair's 32 keys ---------------------
            float lmax[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int pp = 0; pp < 2; ++pp) {
                        const bool page_all = (kbase[pp] + kPageSize - 1) <= min_lim;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int kpos = kbase[pp] + fp8_key_of_row(g + 8 * h);
                            float v = s[pp][nt][2 * h + e] * sl2;
                            if (pp == 1 && !two) {
                                v = -INFINITY;
                            } else if (!page_all) {
                                bool allow = kpos <= lim[nt][e];
                                if (!allow && kpos >= prefix && kpos < si.seq_len)
                                    allow = (anc[nt][e] >> (kpos - prefix)) & 1ull;
                                v = allow ? v : -INFINITY;
                            }
                            s[pp][nt][2 * h + e] = v;
                            mx = fmaxf(mx, v);
                        }
                    }
                    lmax[nt][e] = mx;
                }
            // -- lazy rescale: only when some score passed its row's reference by the slack (or
            //    the row has no reference yet); the row max (shuffles) only in that case --------
            bool need = false;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    need |= lmax[nt][e] > mref[nt][e] + kRescaleSlack ||
                            (mref[nt][e] == -INFINITY && lmax[nt][e] != -INFINITY);
            if (__any_sync(0xffffffffu, need)) {
                float cmax[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float mx = lmax[nt][e];
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        cmax[nt][e] = mx;
                    }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float mnew = fmaxf(mref[nt][e], cmax[nt][e]);
                        if (mnew != mref[nt][e]) {
                            const float alpha = mref[nt][e] == -INFINITY ? 0.f : exp2f(mref[nt][e] - mnew);
                            mref[nt][e] = mnew;
                            lsum[nt][e] *= alpha;
#pragma unroll
                            for (int dt = 0; dt < KS; ++dt) {
                                o[dt][nt][e] *= alpha;
                                o[dt][nt][2 + e] *= alpha;
                            }
                        }
                    }
            }
            // -- P = exp2(S - ref) in f16, row sums, P^T by an in-register transpose ----------
            uint32_t pb[2][NT][2];
#pragma unroll
            for (int pp = 0; pp < 2; ++pp)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float pv[4];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float ref = mref[nt][e] == -INFINITY ? 0.f : mref[nt][e];
                        pv[e] = exp2f(s[pp][nt][e] - ref);
                        pv[2 + e] = exp2f(s[pp][nt][2 + e] - ref);
                        lsum[nt][e] += pv[e] + pv[2 + e];
                    }
                    pb[pp][nt][0] = movmatrix_trans(pack_f16x2(pv[0], pv[1]));   // M rows 0..7
                    pb[pp][nt][1] = movmatrix_trans(pack_f16x2(pv[2], pv[3]));   // M rows 8..15
                }
            // slots past the sequence's end hold stale codes (NaN among them): zero those V
            // bytes so that P = 0 times a non-finite value cannot reach the accumulators. In a
            // transposed page, byte j of each 16-byte head-dim row is key j.
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                if (pp == 1 && !two) break;
                const int nvalid = si.seq_len - kbase[pp];
                if (nvalid < kPageSize) {
                    for (int d = lane; d < D; d += 32) {
                        uint4* rowp = reinterpret_cast<uint4*>(Vp[pp] + d * kPageSize);
                        uint4 v = *rowp;
                        uint32_t* wv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int keep = min(max(nvalid - 4 * q4, 0), 4);   // bytes of this word to keep
                            wv[q4] &= keep >= 4 ? 0xffffffffu : ((1u << (8 * keep)) - 1u);
                        }
                        *rowp = v;
                    }
                    __syncwarp();
                }
            }
            // -- O^T += V^T P^T for both pages ----------------------------------------------
#pragma unroll
            for (int d2 = 0; d2 < KS; d2 += 2) {
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    if (pp == 1 && !two) break;
                    // head-dim rows 16 d2 + (0..31) of the transposed page, 16 key bytes each
                    uint32_t r[4];
                    ldmatrix_x4(r, Vp[pp] + (16 * d2 + v8_row) * kPageSize);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        uint32_t a[4];
                        e4m3x4_to_f16x2x2(r[2 * kk], a[0], a[2]);
                        e4m3x4_to_f16x2x2(r[2 * kk + 1], a[1], a[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_f16_16816(o[d2 + kk][nt], a, pb[pp][nt]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                fence_proxy_async_smem();
#pragma unroll
                for (int pp = 0; pp < 2; ++pp)
                    if ((pp == 0 || two) && i + pp + C::NS < n_my)
                        issue_page<D, C::NS, C::STAGE_BYTES, C::PAGE_BYTES, NW, FP8>(p, w, bts, ring, bar, warp,
                                                                                  i + pp + C::NS, &tmK, &tmV);
            }
        }
    } else {
        for (int i = 0; i < n_my; ++i) {
            const int stage = i % C::NS;
            const bool got = mbar_wait_bounded(&bar[stage], (i / C::NS) & 1, p.err, PKVA_DEVERR_TIMEOUT);
            waited = i + 1;
            if (__any_sync(0xffffffffu, !got)) {
                ok = false;
                break;
            }
            uint8_t* Ks = ring + stage * C::STAGE_BYTES;
            uint8_t* Vs = Ks + C::PAGE_BYTES;
            const int kbase = (w.page_begin + warp + NW * i) * kPageSize;
            if constexpr (!FP8) {
                if (p.append && kbase + kPageSize > prefix && kbase < si.seq_len) {
                    // fused append: the new tokens' rows come from the dense input, not the cache
                    const int r0 = max(prefix - kbase, 0), r1 = min(si.seq_len - kbase, kPageSize);
                    patch_page_rows<D>(Ks, Vs, p.k_new, p.v_new, si, p.Hkv, w.kv_head, r0, r1, kbase + r0 - prefix,
                                       lane);
                    __syncwarp();
                }
            }

            bf16_page<D, NT, C::QB>(Ks, Vs, qs, qf, kbase, prefix, si.seq_len, min_lim, lim, anc, sl2, o, mref, lsum);
            __syncwarp();
            if (lane == 0 && i + C::NS < n_my) {
                fence_proxy_async_smem();
                issue_page<D, C::NS, C::STAGE_BYTES, C::PAGE_BYTES, NW, FP8>(p, w, bts, ring, bar, warp, i + C::NS,
                                                                          &tmK, &tmV);
            }
        }
    }
    if (!ok) {
        for (int i = waited; i < n_my && i < waited + C::NS; ++i)
            mbar_wait_bounded(&bar[i % C::NS], (i / C::NS) & 1, p.err, PKVA_DEVERR_TIMEOUT);
        if (lane == 0) atomicOr(&flag[1], 1);
    }
    __syncwarp();
    if (warp < NW && lane == 0)                    // every phase of this warp's stages is complete
        for (int i = 0; i < C::NS; ++i) mbar_inval(&bar[i]);
    if constexpr (FP8) {                           // the V scale of this KV head
        const float vs = p.v_scale[w.kv_head];
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[dt][nt][e] *= vs;
    }
    // row sums over the 16 keys: lanes with the same t4 hold the column
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = lsum[nt][e];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            lsum[nt][e] = l;
        }

    grp.sync();
    float* cm = reinterpret_cast<float*>(sm);       // [NW][NR]
    float* cl = cm + NW * NR;                       // [NW][NR]
    float* co = cl + NW * NR;                       // [NW][NR][D]
    if (warp < NW && g == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int c = nt * 8 + 2 * t4 + e;
                cm[warp * NR + c] = mref[nt][e];
                cl[warp * NR + c] = lsum[nt][e];
            }
    }
    if (warp < NW) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int dt = 0; dt < KS; ++dt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = nt * 8 + 2 * t4 + (i & 1);
                    const int d = dt * 16 + g + 8 * (i >> 1);
                    co[(warp * NR + c) * D + d] = o[dt][nt][i];
                }
    }
    grp.sync();
    merge_and_store<D, NR, NW>(grp, p, w, cm, cl, co, rout, flag);
    if (p.append && w.row_begin == 0 && w.split <= 0) {          // one task per (sequence, KV head)
        if constexpr (FP8)
            append_rows_fp8<D>(p.k_new, p.v_new, reinterpret_cast<uint8_t*>(p.k_cache),
                               reinterpret_cast<uint8_t*>(p.v_cache), p.block_table, p.bt_stride, p.num_pages, p.Hkv,
                               p.err, si, w.seq, w.kv_head, 0, si.query_len, tid, grp.n, p.k_scale[w.kv_head],
                               p.v_scale[w.kv_head]);
        else
            append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages, p.Hkv,
                           p.err, si, w.seq, w.kv_head, 0, si.query_len, tid, grp.n);
    }
}

// =====================================================================================
// Row-split (wide) task: one pass over the pages for up to 48 packed rows.
// =====================================================================================
// A verify unit of a (sequence, KV head) has T draft tokens x G query heads packed rows
// (5 x 7 = 35 on the Qwen2-7B shape), more than the 16 columns one warp's tiles hold. The
// page-streaming task above would take such a unit as several 16-row tasks that each read
// every page of the unit again. Here one task takes up to three 16-row chunks of the unit:
// warp 3 streams each page once through a ring shared by the task (TMA, a full and an
// empty mbarrier per stage), and warps 0..2 each run the page body for their own chunk on
// every page, so no warp shares rows with another and nothing is combined across warps.
// Every chunk keeps its own split unit (partial slots, arrival counter), so splits and
// shared-prefix partials work per chunk as for the page-streaming task.
constexpr int kWideChunks = 3;                           // consumer warps (16-row chunks)
constexpr int kWideRows = kWideChunks * kDecodeRowsMax;  // rows one wide task holds
constexpr int kWideProducer = 3;                         // the warp that issues the page loads

// Shared-memory bytes of a wide task with `nsw` ring stages (the map of WideCfg).
constexpr int wide_bytes(int D, int nsw) {
    return align_up(align_up(align_up(nsw * 2 * kPageSize * D * 2 + kWideRows * 4, 8) + kWideRows * 12, 8) +
                        2 * nsw * 8 + 48, 128) + kWideRows * D * 2;
}

// The most ring stages a wide task can have within `budget` bytes of shared memory.
constexpr int wide_stages(int D, int budget) {
    int n = 1;
    while (n < 32 && wide_bytes(D, n + 1) <= budget) ++n;
    return n;
}

template <int D, int NSW_>
struct WideCfg {
    static constexpr int NSW = NSW_;                      // ring stages (one page each)
    static constexpr int PAGE_BYTES = kPageSize * D * 2;
    static constexpr int STAGE_BYTES = 2 * PAGE_BYTES;    // K page + V page
    static constexpr int RING = NSW * STAGE_BYTES;
    static constexpr int OFF_LIM = RING;
    static constexpr int OFF_ANC = align_up(OFF_LIM + kWideRows * 4, 8);
    static constexpr int OFF_OUT = OFF_ANC + kWideRows * 8;
    static constexpr int OFF_BAR = align_up(OFF_OUT + kWideRows * 4, 8);   // full[NSW], empty[NSW]
    static constexpr int OFF_FLAG = OFF_BAR + 2 * NSW * 8;   // [0, 3) merge flags, [3] units to merge,
                                                             // [4, 7) their ids, [8, 11) row offsets
    static constexpr int OFF_Q = align_up(OFF_FLAG + 48, 128);
    static constexpr int BYTES = OFF_Q + kWideRows * D * 2;
    static_assert(kWideRows * (D + 2) * 4 <= RING, "end-of-task buffers must fit in the ring");
    static_assert(BYTES == wide_bytes(D, NSW), "wide task map");
};

template <int D, int NSW>
__device__ __forceinline__ void decode_wide_task(const Group& grp, const DecodeParams& p, int task,
                                                 const CUtensorMap& tmK, const CUtensorMap& tmV, uint8_t* sm) {
    using C = WideCfg<D, NSW>;
    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const DecodeWork w = p.work[task];
    const SeqInfo si = p.seqs[w.seq];
    const int R = w.row_count;                               // 17 .. 48
    const int nch = (R + kDecodeRowsMax - 1) / kDecodeRowsMax;
    const int npg = w.page_end - w.page_begin;
    const int prefix = si.seq_len - si.query_len;

    int* rlim = reinterpret_cast<int*>(sm + C::OFF_LIM);
    uint64_t* ranc = reinterpret_cast<uint64_t*>(sm + C::OFF_ANC);
    int* rout = reinterpret_cast<int*>(sm + C::OFF_OUT);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint64_t* empty = full + NSW;
    int* flag = reinterpret_cast<int*>(sm + C::OFF_FLAG);
    uint8_t* qs = sm + C::OFF_Q;
    uint8_t* ring = sm;

    if (tid == 0) {
        for (int i = 0; i < NSW; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], nch);
        }
        fence_mbar_init();
        fence_proxy_async_smem();                 // the block's earlier generic accesses come first
        for (int i = 0; i < 12; ++i) flag[i] = 0;
    }
    // per-row records: output row, causal limit, tree ancestor mask
    for (int r = tid; r < kWideRows; r += grp.n) {
        if (r < R) {
            const int t = (w.row_begin + r) / p.G;
            rout[r] = q_row_index(p, si, w, r);
            rlim[r] = si.mask_kind == PKVA_CAUSAL ? prefix + t : prefix - 1;
            ranc[r] = si.mask_kind == PKVA_CAUSAL ? 0ull : p.anc[si.anc_off + t];
        } else {
            rout[r] = -1;
            rlim[r] = 0x7fffffff;
            ranc[r] = 0ull;
        }
    }
    // Q rows staged in shared memory (16-byte chunk c of row r at c ^ (r & 7)); missing rows zero
    for (int idx = tid; idx < kWideRows * (D / 8); idx += grp.n) {
        const int r = idx / (D / 8), c = idx - r * (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < R) v = *reinterpret_cast<const uint4*>(p.q + (int64_t)q_row_index(p, si, w, r) * D + c * 8);
        *reinterpret_cast<uint4*>(qs + r * (D * 2) + ((c ^ (r & 7)) << 4)) = v;
    }
    grp.sync();

    bool ok = true;
    if (warp == kWideProducer) {
        // ---- producer: every page once, in order; a stage is refilled once all chunks are done
        //      with it. Block-table entries are read 32 at a time and handed out by shuffle.
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const int32_t* btrow = p.block_table + (int64_t)w.seq * p.bt_stride + w.page_begin;
        int issued = 0;
        for (int base = 0; base < npg && ok; base += 32) {
            int ph = -1;
            if (base + lane < npg) {
                ph = btrow[base + lane];
                if (ph < 0 || ph >= p.num_pages) {
                    atomicOr(p.err, PKVA_DEVERR_BAD_PAGE);
                    ph = -1;                      // read from a fully out-of-bounds box: zeros
                }
            }
            const int n = min(32, npg - base);
            for (int j = 0; j < n; ++j) {
                const int phj = __shfl_sync(0xffffffffu, ph, j);
                const int i = base + j;
                bool got = true;
                if (lane == 0) {
                    if (i >= NSW)
                        got = mbar_wait_bounded(&empty[i % NSW], ((i / NSW) - 1) & 1, p.err, PKVA_DEVERR_TIMEOUT);
                    if (got) {
                        fence_proxy_async_smem();
                        issue_page_at<D, NSW, C::STAGE_BYTES, C::PAGE_BYTES>(p, w, phj, ring, full, i, &tmK, &tmV);
                    }
                }
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                ++issued;
            }
        }
        // every issued load has landed before the ring is reused (the consumers normally
        // waited for all of them already)
        if (lane == 0)
            for (int i = max(0, issued - NSW); i < issued; ++i)
                mbar_wait_bounded(&full[i % NSW], (i / NSW) & 1, p.err, PKVA_DEVERR_TIMEOUT);
        __syncwarp();
    }

    // ---- consumers: warp c owns packed rows [16c, 16c + 16) of the task
    constexpr int NT = 2;
    constexpr int KS = D / 16;
    float o[KS][NT][4];
    float mref[NT][2], lsum[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            mref[nt][e] = -INFINITY;
            lsum[nt][e] = 0.f;
        }
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[dt][nt][i] = 0.f;
    }
    const bool consumer = warp < nch;
    if (consumer) {
        const int r0 = warp * kDecodeRowsMax;
        int lim[NT][2];
        uint64_t anc[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int c = r0 + nt * 8 + 2 * t4 + e;
                lim[nt][e] = rlim[c];
                anc[nt][e] = ranc[c];
            }
        int min_lim = 0x7fffffff;
        for (int r = r0; r < min(R, r0 + kDecodeRowsMax); ++r) min_lim = min(min_lim, rlim[r]);
        const uint8_t* qw = qs + r0 * (D * 2);
        const uint32_t qf_unused[NT][1][2] = {};
        const float sl2 = p.scale_log2;
        for (int i = 0; i < npg; ++i) {
            const int stage = i % NSW;
            const bool got = mbar_wait_bounded(&full[stage], (i / NSW) & 1, p.err, PKVA_DEVERR_TIMEOUT);
            if (__any_sync(0xffffffffu, !got)) {
                ok = false;
                break;
            }
            uint8_t* Ks = ring + stage * C::STAGE_BYTES;
            uint8_t* Vs = Ks + C::PAGE_BYTES;
            const int kbase = (w.page_begin + i) * kPageSize;
            if (p.append && kbase + kPageSize > prefix && kbase < si.seq_len) {
                // fused append: the new tokens' rows come from the dense input (each chunk's warp
                // writes the same bytes, so the copies agree whichever lands last)
                const int a0 = max(prefix - kbase, 0), a1 = min(si.seq_len - kbase, kPageSize);
                patch_page_rows<D>(Ks, Vs, p.k_new, p.v_new, si, p.Hkv, w.kv_head, a0, a1, kbase + a0 - prefix,
                                   lane);
                __syncwarp();
            }
            bf16_page<D, NT, true>(Ks, Vs, qw, qf_unused, kbase, prefix, si.seq_len, min_lim, lim, anc, sl2, o,
                                   mref, lsum);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        // row sums over the 16 keys: lanes with the same t4 hold the column
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float l = lsum[nt][e];
                l += __shfl_xor_sync(0xffffffffu, l, 4);
                l += __shfl_xor_sync(0xffffffffu, l, 8);
                l += __shfl_xor_sync(0xffffffffu, l, 16);
                lsum[nt][e] = l;
            }
    }
    grp.sync();                                     // every page consumed and every load landed
    if (tid == 0)
        for (int i = 0; i < NSW; ++i) {
            mbar_inval(&full[i]);
            mbar_inval(&empty[i]);
        }

    // ---- per-row state into shared memory (the ring is free now) --------------------
    float* cm = reinterpret_cast<float*>(sm);       // [48]
    float* cl = cm + kWideRows;                     // [48]
    float* co = cl + kWideRows;                     // [48][D]
    if (consumer) {
        const int r0 = warp * kDecodeRowsMax;
        if (g == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = r0 + nt * 8 + 2 * t4 + e;
                    cm[c] = mref[nt][e];
                    cl[c] = lsum[nt][e];
                }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int dt = 0; dt < KS; ++dt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = r0 + nt * 8 + 2 * t4 + (i & 1);
                    const int d = dt * 16 + g + 8 * (i >> 1);
                    co[c * D + d] = o[dt][nt][i];
                }
    }
    grp.sync();

    // ---- rows out, or each chunk's partial into its unit's slot ----------------------
    const bool split = w.unit >= 0;
    for (int idx = tid; idx < R * (D / 2); idx += grp.n) {
        const int r = idx / (D / 2);
        const int c = (idx - r * (D / 2)) * 2;
        const float2 v = *reinterpret_cast<const float2*>(co + r * D + c);
        if (!split) {
            const float L = cl[r];
            const float inv = L > 0.f ? 1.f / L : 0.f;
            *reinterpret_cast<__nv_bfloat162*>(p.out + (int64_t)rout[r] * D + c) =
                __floats2bfloat162_rn(v.x * inv, v.y * inv);
        } else {
            const int ch = r / kDecodeRowsMax, rr = r - ch * kDecodeRowsMax;
            const int slot = p.units[w.unit + ch].slot_base + w.split;
            *reinterpret_cast<float2*>(p.part_o + ((int64_t)slot * kDecodeRowsMax + rr) * D + c) = v;
            if (c == 0)
                *reinterpret_cast<float2*>(p.part_ml + ((int64_t)slot * kDecodeRowsMax + rr) * 2) =
                    make_float2(cm[r], cl[r]);
        }
    }
    if (split) {
        // ---- split-KV combine per chunk: the last task of a unit to finish merges it ------
        __threadfence();
        grp.sync();
        if (tid < nch) {
            const int u = w.unit + tid;
            const int prev = atomicAdd(&p.counters[u], 1);
            flag[tid] = (prev == p.units[u].arrivals - 1);
            if (flag[tid]) p.counters[u] = 0;           // every arrival is in: ready for the next run
        }
        grp.sync();
        if (tid == 0) {
            int n = 0, rows = 0;
            for (int ch = 0; ch < nch; ++ch)
                if (flag[ch]) {
                    flag[4 + n] = w.unit + ch;
                    flag[8 + n] = rows;
                    rows += p.units[w.unit + ch].row_count;
                    ++n;
                }
            flag[3] = n;
            flag[11] = rows;
        }
        grp.sync();
        if (flag[3] > 0) {
            __threadfence();
            merge_units<D>(warp, grp.n >> 5, lane, flag + 4, flag + 8, flag[3], flag[11], p.units, p.part_o,
                           p.part_ml, p.seqs, p.out, p.Hq, p.G);
        }
    }
    if (p.append && w.row_begin == 0 && w.split <= 0)          // one task per (sequence, KV head)
        append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages, p.Hkv,
                       p.err, si, w.seq, w.kv_head, 0, si.query_len, tid, grp.n);
}

// =====================================================================================
// CUDA-core page body (fp32 FMA).
// =====================================================================================
// One decode/verify task on the CUDA-core page body (all NW warps stream pages).
template <int D, int NR, int NW, int NS>
__device__ __forceinline__ void decode_fma_task(const Group& grp, const DecodeParams& p, int task,
                                                const CUtensorMap& tmK, const CUtensorMap& tmV, uint8_t* sm) {
    using C = DecodeCfg<D, NR, true, NW, NS>;

    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const DecodeWork w = p.work[task];
    const SeqInfo si = p.seqs[w.seq];

    float* qs = reinterpret_cast<float*>(sm + C::OFF_Q);
    float* ps = reinterpret_cast<float*>(sm + C::OFF_P);
    int* bts = reinterpret_cast<int*>(sm + C::OFF_BT);
    int* rlim = reinterpret_cast<int*>(sm + C::OFF_LIM);
    uint64_t* ranc = reinterpret_cast<uint64_t*>(sm + C::OFF_ANC);
    int* rout = reinterpret_cast<int*>(sm + C::OFF_OUT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    int* flag = reinterpret_cast<int*>(sm + C::OFF_FLAG);

    const int R = w.row_count;
    const int npg = w.page_end - w.page_begin;
    const int prefix = si.seq_len - si.query_len;

    task_setup<NR, C::NS, NW>(grp, p, w, si, bts, rlim, ranc, rout, bars, flag, &tmK, &tmV);
    // Q rows in fp32, pre-scaled by scale*log2(e); each row is stored as two halves with a
    // 4-float pad so that the two lane halves read different banks
    for (int idx = tid; idx < NR * (D / 8); idx += grp.n) {
        const int r = idx / (D / 8);
        const int c8 = (idx - r * (D / 8)) * 8;
        float f[8];
        if (r < R) {
            const uint4 raw = *reinterpret_cast<const uint4*>(p.q + (int64_t)q_row_index(p, si, w, r) * D + c8);
            bf16x8_to_f32(raw, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= p.scale_log2;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.f;
        }
        const int hh = c8 / C::HALF;
        float* dst = qs + r * C::QROW + hh * (C::HALF + 4) + (c8 - hh * C::HALF);
        *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
    grp.sync();

    int min_lim = 0x7fffffff;
    for (int r = 0; r < R; ++r) min_lim = min(min_lim, rlim[r]);

    const int n_my = (warp < NW && npg > warp) ? (npg - warp + NW - 1) / NW : 0;
    uint8_t* ring = sm + warp * C::NS * C::STAGE_BYTES;    // used only by warps < NW
    uint64_t* bar = bars + warp * C::NS;

    float o[NR][C::OPL];
    float m_run[NR], l_run[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        m_run[r] = -INFINITY;
        l_run[r] = 0.f;
#pragma unroll
        for (int c = 0; c < C::OPL; ++c) o[r][c] = 0.f;
    }

    if (lane == 0)
        for (int i = 0; i < C::NS && i < n_my; ++i)
            issue_page<D, C::NS, C::STAGE_BYTES, C::PAGE_BYTES, NW>(p, w, bts, ring, bar, warp, i, &tmK, &tmV);
    __syncwarp();

    const int j = lane & 15;       // key slot of this lane in the QK phase
    const int hh = lane >> 4;      // which half of the head dimension it sums
    float* pw = ps + warp * kPageSize * NR;
    bool ok = true;
    int waited = 0;

    for (int i = 0; i < n_my; ++i) {
        const int stage = i % C::NS;
        const bool got = mbar_wait_bounded(&bar[stage], (i / C::NS) & 1, p.err, PKVA_DEVERR_TIMEOUT);
        waited = i + 1;
        if (__any_sync(0xffffffffu, !got)) {
            ok = false;
            break;
        }
        uint8_t* Ks = ring + stage * C::STAGE_BYTES;
        uint8_t* Vs = Ks + C::PAGE_BYTES;
        const int kbase = (w.page_begin + warp + NW * i) * kPageSize;
        if (p.append && kbase + kPageSize > prefix && kbase < si.seq_len) {
            const int r0 = max(prefix - kbase, 0), r1 = min(si.seq_len - kbase, kPageSize);
            patch_page_rows<D>(Ks, Vs, p.k_new, p.v_new, si, p.Hkv, w.kv_head, r0, r1, kbase + r0 - prefix, lane);
            __syncwarp();
        }

        // -- scores: lane (j, hh) sums half hh of <q_r, k_j> for every row r ------------
        float acc[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) acc[r] = 0.f;
#pragma unroll
        for (int cc = 0; cc < C::HALF / 8; ++cc) {
            const int col = hh * C::HALF + cc * 8;
            const int box = col >> 6, ch = (col & 63) >> 3;
            const uint4 kr = *reinterpret_cast<const uint4*>(Ks + box * kBoxBytes + j * 128 + ((ch ^ (j & 7)) << 4));
            float kf[8];
            bf16x8_to_f32(kr, kf);
            const float* qp = qs + hh * (C::HALF + 4) + cc * 8;
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                if (r < R) {
                    const float4 a = *reinterpret_cast<const float4*>(qp + r * C::QROW);
                    const float4 b = *reinterpret_cast<const float4*>(qp + r * C::QROW + 4);
                    float t = acc[r];
                    t = fmaf(kf[0], a.x, t);
                    t = fmaf(kf[1], a.y, t);
                    t = fmaf(kf[2], a.z, t);
                    t = fmaf(kf[3], a.w, t);
                    t = fmaf(kf[4], b.x, t);
                    t = fmaf(kf[5], b.y, t);
                    t = fmaf(kf[6], b.z, t);
                    t = fmaf(kf[7], b.w, t);
                    acc[r] = t;
                }
            }
        }
        // -- mask, online softmax (warp-shuffle max over the page's 16 keys) --------------
        const int kpos = kbase + j;
        const bool page_all = (kbase + kPageSize - 1) <= min_lim;
        float alpha[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            alpha[r] = 1.f;
            if (r < R) {
                float s = acc[r] + __shfl_xor_sync(0xffffffffu, acc[r], 16);
                bool allow = page_all || kpos <= rlim[r];
                if (!allow && kpos >= prefix && kpos < si.seq_len)
                    allow = (ranc[r] >> (kpos - prefix)) & 1ull;
                s = allow ? s : -INFINITY;
                float mx = s;
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                const float mnew = fmaxf(m_run[r], mx);
                const float ref = (mnew == -INFINITY) ? 0.f : mnew;
                const float pr = exp2f(s - ref);
                alpha[r] = exp2f(m_run[r] - ref);
                m_run[r] = mnew;
                l_run[r] = fmaf(l_run[r], alpha[r], pr);
                acc[r] = pr;
            } else {
                acc[r] = 0.f;
            }
        }
        if (hh == 0) {
#pragma unroll
            for (int r4 = 0; r4 < NR / 4; ++r4)
                *reinterpret_cast<float4*>(pw + j * NR + 4 * r4) =
                    make_float4(acc[4 * r4], acc[4 * r4 + 1], acc[4 * r4 + 2], acc[4 * r4 + 3]);
        }
        __syncwarp();

        // -- o_r = alpha_r * o_r + sum_j p_rj v_j; lane owns D/32 output columns ------------
#pragma unroll
        for (int r = 0; r < NR; ++r)
            if (r < R)
#pragma unroll
                for (int c = 0; c < C::OPL; ++c) o[r][c] *= alpha[r];
        const int nvalid = min(kPageSize, si.seq_len - kbase);   // slots past L are skipped
#pragma unroll 4
        for (int jj = 0; jj < nvalid; ++jj) {
            float vf[C::OPL];
            if constexpr (D == 128) {
                const int box = lane >> 4, ch = (lane & 15) >> 1;
                const uint2 vr = *reinterpret_cast<const uint2*>(Vs + box * kBoxBytes + jj * 128 +
                                                                 ((ch ^ (jj & 7)) << 4) + (lane & 1) * 8);
                bf16x2_to_f32(vr.x, vf[0], vf[1]);
                bf16x2_to_f32(vr.y, vf[2], vf[3]);
            } else {
                const int ch = lane >> 2;
                const uint32_t vr = *reinterpret_cast<const uint32_t*>(Vs + jj * 128 + ((ch ^ (jj & 7)) << 4) +
                                                                       (lane & 3) * 4);
                bf16x2_to_f32(vr, vf[0], vf[1]);
            }
#pragma unroll
            for (int r4 = 0; r4 < NR / 4; ++r4) {
                const float4 pp = *reinterpret_cast<const float4*>(pw + jj * NR + 4 * r4);
                const float pv[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = 4 * r4 + e;
                    if (r < R)
#pragma unroll
                        for (int c = 0; c < C::OPL; ++c) o[r][c] = fmaf(pv[e], vf[c], o[r][c]);
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + C::NS < n_my) {
            fence_proxy_async_smem();
            issue_page<D, C::NS, C::STAGE_BYTES, C::PAGE_BYTES, NW>(p, w, bts, ring, bar, warp, i + C::NS, &tmK,
                                                                 &tmV);
        }
    }
    if (!ok) {
        for (int i = waited; i < n_my && i < waited + C::NS; ++i)
            mbar_wait_bounded(&bar[i % C::NS], (i / C::NS) & 1, p.err, PKVA_DEVERR_TIMEOUT);
        if (lane == 0) atomicOr(&flag[1], 1);
    }

    // row sums: lanes j and j+16 hold the same keys, so reduce within each half
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        float l = l_run[r];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l_run[r] = l;
    }

    grp.sync();
    float* cm = reinterpret_cast<float*>(sm);       // [NW][NR] running max (log2 units)
    float* cl = cm + NW * NR;                       // [NW][NR] running sum
    float* co = cl + NW * NR;                       // [NW][NR][D] unnormalised output
    if (warp < NW && lane == 0) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            cm[warp * NR + r] = m_run[r];
            cl[warp * NR + r] = l_run[r];
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (warp < NW && r < R) {
            float* dst = co + (warp * NR + r) * D + lane * C::OPL;
            if constexpr (C::OPL == 4)
                *reinterpret_cast<float4*>(dst) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
            else
                *reinterpret_cast<float2*>(dst) = make_float2(o[r][0], o[r][1]);
        }
    }
    grp.sync();
    merge_and_store<D, NR, NW>(grp, p, w, cm, cl, co, rout, flag);
    if (p.append && w.row_begin == 0 && w.split <= 0)   // one task per (sequence, KV head)
        append_rows<D>(p.k_new, p.v_new, p.k_cache, p.v_cache, p.block_table, p.bt_stride, p.num_pages, p.Hkv,
                       p.err, si, w.seq, w.kv_head, 0, si.query_len, tid, grp.n);
}


}  // namespace dec
}  // namespace pkva
