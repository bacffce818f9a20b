// gad_prefill_tc.cuh - prefill blocks (many new tokens per request) on the
// 5th-generation tensor cores.
//
// Method: the attention of the page "Prefill layer (muse_prefill_layer)",
// section "What to compute" (QK-norm, RoPE, fp8 cache write, attention,
// rmsnorm(a) * sigmoid(g)), which is the decode page's step ("Gated attention
// decode (muse_attention_decode)", section "What to compute") with q_len 753
// or 16,384, causal within the block.
//
// Items.  A request's L tokens are cut into chunks of PF_CHUNK = 32; an item
// is (request, chunk, KV head g), and its key range is the union of its 32
// tokens' ranges.  The persistent tile list, partial slots and combine step
// are those of the decode kernels (gad_kernels.cuh); a partial row block holds
// 32 tokens x the 8 query heads of KV head g.
//
// Rows.  Two softmax warpgroups each own one 128-row MMA tile of the item:
// warpgroup w holds tokens 16w .. 16w + 15, row r = token 16w + r / 8, query
// head 8g + r % 8.  Both tiles read the same K and V tiles, so one gathered
// and converted 64-key tile feeds 256 rows:
//   S_w = Q_w . K^T     M 128, N 64 keys, K 64 dims   (A = Q_w in tensor memory)
//   O_w += P_w . V      M 128, N 64 dims, K 64 keys   (A = P_w in tensor memory)
// with no padding of the contraction (the verify kernel pads it to 128 to put
// both KV heads in one tile).
//
// Warps: 0-3 softmax of tile 0, 4-7 softmax of tile 1, 8-9 loaders (cp.async
// gathers of the 64-byte K and V halves of KV head g from each cache row,
// E4M3 -> fp16 into 128-byte-swizzled tiles), 10 MMA issue.  Eleven warps
// leave 168 registers per thread (three warps on a scheduler).  Softmax: one
// thread per row; at an item's first tile it writes its row of Q_w into
// tensor memory; per tile S from tensor memory, mask, online softmax with lazy
// rescaling of O in tensor memory, P (fp16) written over the first half of
// its S buffer.  The two warpgroups run their exponentials side by side
// (taking turns on them, so that one's S load, mask and max overlapped the
// other's exponentials, measured 4-5% slower).
// Every
// mbarrier wait is bounded; an expired wait sets the step's error word and
// the CTA winds down, waits for its MMAs and frees its tensor memory.
#pragma once

#include "gad_kernels.cuh"
#include "gad_tc.cuh"

namespace gad {
namespace ptc {

// Which exponentials of the softmax run on the FMA pipe (exp2_poly): the
// second weight of every POLY_EVERY-th pair of keys, 1 in 8 of them.  Measured
// on B200 (kernel us, prefill1_full / 16,384 tokens on 32K): none 647.8 /
// 5,201.8; 1 in 8 638.0 / 5,019.4; 1 in 4 641.9 / 5,088.6; 1 in 2 699.8 /
// 5,705.6 (the FMA pipe also carries the softmax's other arithmetic).
constexpr int POLY_EVERY = 4;

constexpr int TK = 64;                       // keys per tile
constexpr int THREADS = 352;                 // 11 warps
constexpr int SM_THREADS = 128;              // one softmax warpgroup
constexpr int LOAD_T0 = 256;                 // first loader thread (warp 8)
constexpr int LOADERS = 64;
constexpr int MMA_WARP = 10;
constexpr int RAW_ROW = 64;                  // bytes of one KV head in a cache row
constexpr int RAW_STAGE = 2 * TK * RAW_ROW;  // 8 KB: 64 K halves then 64 V halves (E4M3)
constexpr int F16_TILE = TK * 128;           // 64 keys x 64 fp16 = 8 KB (128-byte rows)
constexpr int F16_BUF = 2 * F16_TILE;        // K tile then V tile: 16 KB
constexpr int NKV = 3;                       // converted K/V buffers: the loader converts tile
                                             // i + 1 while P.V of tile i - 1 still reads its own
constexpr uint32_t TM_COLS = 512;            // tensor-memory columns allocated
constexpr uint32_t TM_Q = 0;                 // Q_w at TM_Q + 32 w (fp16 pairs, 32 columns)
constexpr uint32_t TM_S = 64;                // S_w buffer b at TM_S + 128 w + 64 b (P aliases its first 32)
constexpr uint32_t TM_O = 320;               // O_w at TM_O + 64 w
constexpr float RESCALE_LOG2 = 8.f;          // lazy rescale threshold (P stays <= 2^8)

// mbarrier indices
constexpr int BAR_KV_READY = 0;   // [NKV] converted K and V tile                    (64 loader arrivals)
constexpr int BAR_KV_FREE = 3;    // [NKV] both P.V of the tile done: buffer free    (MMA commit)
constexpr int BAR_S_FULL = 6;     // [w][2] S_w of the tile in tensor memory         (MMA commit)
constexpr int BAR_P_FULL = 10;    // [w][2] P_w of the tile in tensor memory         (128 arrivals)
constexpr int BAR_O_FREE = 14;    // [w] O_w read out at an item's last tile         (128 arrivals)
constexpr int BAR_MMA_DONE = 16;  // teardown: all MMAs done                         (MMA commit)
constexpr int BAR_Q_READY = 17;   // [w] Q_w of the item in tensor memory            (128 arrivals)
constexpr int NBARS = 19;

template <int NS>
struct Cfg {
    static constexpr size_t F16_BYTES = NKV * F16_BUF;
    static constexpr size_t RAW_BYTES = static_cast<size_t>(NS) * RAW_STAGE;
    static constexpr int IDX_SLOTS = 2 * NS;
    static constexpr size_t IDX_BYTES = static_cast<size_t>(IDX_SLOTS) * TK * 4;
    static constexpr size_t CTRL_BYTES = 256;  // barriers, tensor-memory base, abort flag
    // + 1024 so the swizzled tiles can start on a 1024-byte boundary
    static size_t smem_bytes(int NB) {
        return 1024 + F16_BYTES + RAW_BYTES + IDX_BYTES + CTRL_BYTES +
               static_cast<size_t>(4 * NB + 1) * 4;
    }
    static_assert(NS >= 3, "stages");
    static_assert(NBARS * 8 + 8 <= static_cast<int>(CTRL_BYTES), "control block");
};


__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = wait_bounded(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace ptc

template <int PS, int NS>
__global__ void __launch_bounds__(ptc::THREADS, 1) prefill_tc_kernel(const StepParams p) {
    using namespace ptc;
    using C = Cfg<NS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* f16 = smem;                                     // [NKV][K, V][64 keys][128 B]
    uint8_t* raw = smem + C::F16_BYTES;                      // [NS][K halves, V halves]
    int* idx_smem = reinterpret_cast<int*>(raw + C::RAW_BYTES);
    uint8_t* ctrl = reinterpret_cast<uint8_t*>(idx_smem) + C::IDX_BYTES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + NBARS * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + NBARS * 8 + 4);
    int* tpre = reinterpret_cast<int*>(ctrl + C::CTRL_BYTES);
    int* rlo = tpre + p.NB + 1;
    int* rhi = rlo + p.NB;
    int* rnew = rhi + p.NB;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int B = p.NB;  // list items (request, chunk, KV head); b below is an item index

    int total, per, t0, t1;
    build_tile_list<TK, true>(p, tpre, rlo, rhi, rnew, THREADS, total, per, t0, t1);
    if (t0 >= t1) return;

    const uint32_t bar0 = smem_addr(ctrl);
    auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    if (tid == 0) {
        for (int b = 0; b < NKV; ++b) {
            mbar_init(BAR(BAR_KV_READY + b), LOADERS);
            mbar_init(BAR(BAR_KV_FREE + b), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(BAR_O_FREE + b), SM_THREADS);
            mbar_init(BAR(BAR_Q_READY + b), SM_THREADS);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(BAR(BAR_S_FULL + i), 1);
            mbar_init(BAR(BAR_P_FULL + i), SM_THREADS);
        }
        mbar_init(BAR(BAR_MMA_DONE), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == MMA_WARP) {
        tc_alloc(smem_addr(tmem_slot), TM_COLS);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- tile cursors over the list (item b owns tiles [tpre[b], tpre[b+1])) ----
    auto find_req = [&](int tau) {
        int lo = 0, hi = B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tpre[mid] <= tau) lo = mid;
            else hi = mid;
        }
        return lo;
    };
    auto advance = [&](int& tau, int& b) {
        ++tau;
        while (b < B - 1 && tau >= tpre[b + 1]) ++b;
    };
    auto tile_k0 = [&](int tau, int b) { return (rlo[b] / TK + (tau - tpre[b])) * TK; };
    const float C2 = __ldg(p.k_scale) * 0.125f * 1.4426950408889634f;  // raw score -> log2 units

    if (warp >= 8 && warp < MMA_WARP) {
        // =================== loaders: gather, convert, A operands ===================
        const int ltid = tid - LOAD_T0;
        bool prep_done = false;
        auto ensure_prep = [&]() {
            if (!prep_done) {
                pdl_wait_primary();
                prep_done = true;
            }
        };
        // A cursor over the tile list that keeps its item's data in registers:
        // shared memory is read only when it enters a new item, and so is the
        // item's request and KV head (integer division by a runtime value runs
        // on the MUFU, which the softmax warps keep busy with exponentials).
        struct Cur {
            int tau, b, end, k0, lo, hi, rnew;
            const int32_t* pt;  // page-table row of the item's request
            size_t gofs;        // byte offset of KV head g in a cache row
        };
        auto cur_enter = [&](Cur& c) {  // c.tau and c.b set
            c.end = tpre[c.b + 1];
            c.lo = rlo[c.b];
            c.hi = rhi[c.b];
            c.rnew = rnew[c.b];
            c.k0 = (c.lo / TK + (c.tau - tpre[c.b])) * TK;
            const ItemRef it = item_ref<true>(p, c.b);
            c.pt = p.page_table + static_cast<size_t>(it.req) * p.max_pages;
            c.gofs = static_cast<size_t>(it.grp) * RAW_ROW;
        };
        auto cur_init = [&](Cur& c, int tau) {
            c.tau = tau;
            c.b = find_req(tau);
            cur_enter(c);
        };
        auto cur_next = [&](Cur& c) {
            ++c.tau;
            c.k0 += TK;
            if (c.tau >= c.end && c.tau < t1 && c.b < B - 1) {
                do {
                    ++c.b;
                } while (c.b < B - 1 && c.tau >= tpre[c.b + 1]);
                cur_enter(c);
            }
        };
        auto issue_idx = [&](const Cur& c) {
            if (c.tau >= t1) return;
            int* dst = idx_smem + ((c.tau - t0) % C::IDX_SLOTS) * TK;
            if (PS == 1) {
                if (ltid < TK) {
                    const int k = c.k0 + ltid;
                    if (k >= c.lo && k <= c.hi && k < p.max_pages) cp_async4(smem_addr(dst + ltid), c.pt + k);
                    else dst[ltid] = -1;
                }
            } else {
                if (ltid < TK / PS) {
                    const int pg = c.k0 / PS + ltid;
                    if (pg < p.max_pages) cp_async4(smem_addr(dst + ltid), c.pt + pg);
                    else dst[ltid] = -1;
                }
            }
        };
        // Tile rows: thread = (16-byte chunk j = ltid % 4, rows ltid / 4 + 16 i) of
        // the 64-byte K and V halves of KV head g, so the 4 chunks of a half row
        // come from consecutive lanes (8 rows per warp instruction).  Raw rows are
        // 64 bytes with chunk j stored at j ^ ((r / 2) & 3): 8 consecutive rows
        // cover all 32 banks for the conversion's reads.
        auto issue_kv = [&](const Cur& c) {
            if (c.tau >= t1) return;
            if (c.k0 + TK - 1 >= c.rnew) ensure_prep();
            const int* ix = idx_smem + ((c.tau - t0) % C::IDX_SLOTS) * TK;
            const uint32_t base = smem_addr(raw + ((c.tau - t0) % NS) * RAW_STAGE);
            const int j = ltid & 3;
            const size_t gofs = c.gofs + j * 16;
            constexpr int ROWS = TK * 4 / LOADERS;  // rows per thread
            // all page-table reads first, then the copies
            int pix[ROWS];
#pragma unroll
            for (int i = 0; i < ROWS; ++i) {
                const int r = (ltid >> 2) + (LOADERS / 4) * i;
                pix[i] = PS == 1 ? ix[r] : ix[r / PS];
            }
#pragma unroll
            for (int i = 0; i < ROWS; ++i) {
                const int r = (ltid >> 2) + (LOADERS / 4) * i;
                const int k = c.k0 + r;
                int64_t crow;
                if (PS == 1) crow = pix[i];
                else crow = pix[i] >= 0 ? static_cast<int64_t>(pix[i]) * PS + r % PS : -1;
                const bool ok = k >= c.lo && k <= c.hi && crow >= 0 && crow < p.num_rows;
                const size_t off = ok ? static_cast<size_t>(crow) * ROWB + gofs : 0;
                const uint32_t d = base + r * RAW_ROW + ((j ^ ((r >> 1) & 3)) << 4);
                cp_async16(d, p.k_cache + off, ok ? 16 : 0);
                cp_async16(d + TK * RAW_ROW, p.v_cache + off, ok ? 16 : 0);
            }
        };
        // raw stage -> fp16 tiles: thread = row r of K and of V; 64 codes -> 8 fp16
        // chunks of a 128-byte row, chunk c stored at c ^ (r & 7).
        auto convert = [&](int stage, int buf) {
            const int r = ltid;
#pragma unroll
            for (int kv = 0; kv < 2; ++kv) {
                const uint32_t src = smem_addr(raw + stage * RAW_STAGE) + kv * TK * RAW_ROW + r * RAW_ROW;
                const uint32_t dst = smem_addr(f16 + buf * F16_BUF) + kv * F16_TILE + r * 128;
                uint4 w[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) w[j] = lds128(src + ((j ^ ((r >> 1) & 3)) << 4));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 a, b;
                    a.x = e4m3x2_to_f16x2(w[j].x);
                    a.y = e4m3x2_to_f16x2(w[j].x >> 16);
                    a.z = e4m3x2_to_f16x2(w[j].y);
                    a.w = e4m3x2_to_f16x2(w[j].y >> 16);
                    b.x = e4m3x2_to_f16x2(w[j].z);
                    b.y = e4m3x2_to_f16x2(w[j].z >> 16);
                    b.z = e4m3x2_to_f16x2(w[j].w);
                    b.w = e4m3x2_to_f16x2(w[j].w >> 16);
                    sts128(dst + (((2 * j) ^ (r & 7)) << 4), a);
                    sts128(dst + (((2 * j + 1) ^ (r & 7)) << 4), b);
                }
            }
        };

        Cur xc, kc;  // page-table cursor (runs NS - 1 tiles ahead), gather cursor
        cur_init(xc, t0);
        kc = xc;
        for (int d = 0; d < NS - 1; ++d) {
            issue_idx(xc);
            cur_next(xc);
        }
        cp_async_commit();
        cp_async_wait<0>();
        bar_red_or(1, LOADERS, false);
        for (int d = 0; d < NS - 1; ++d) {
            issue_kv(kc);
            cur_next(kc);
            issue_idx(xc);
            cur_next(xc);
            cp_async_commit();
        }
        const int n_tiles = t1 - t0;
        for (int i = 0; i < n_tiles; ++i) {
            cp_async_wait<NS - 2>();
            bool bad = false;
            // buffer i % NKV is free once both P.V of tile i - NKV are done
            if (i >= NKV) bad = !wait_bounded(BAR(BAR_KV_FREE + i % NKV), (i / NKV - 1) & 1, abort_flag);
            // past this barrier: tile i landed for every loader, and every loader
            // has converted tile i - 1, so its raw stage may be refilled
            if (bar_red_or(1, LOADERS, bad)) break;
            convert(i % NS, i % NKV);
            fence_proxy_async_smem();
            mbar_arrive(BAR(BAR_KV_READY + i % NKV));
            issue_kv(kc);
            cur_next(kc);
            issue_idx(xc);
            cur_next(xc);
            cp_async_commit();
        }
        cp_async_wait<0>();
    }
    else if (warp == MMA_WARP) {
        // =================== MMA issue (whole warp, one elected lane issues) ===================
        constexpr uint32_t ID_S = idesc_f16_f32(128, TK, 0);  // S_w: Q_w . K^T, K-major B
        constexpr uint32_t ID_O = idesc_f16_f32(128, 64, 1);  // O_w: P_w . V, MN-major B
        const uint32_t f16_base = smem_addr(f16);
        // O_w += P_w(k) . V(k) for both tiles; the commit frees the tile's buffers.
        auto issue_pv = [&](int k, bool first, int seg) {
            const uint32_t vbuf = f16_base + (k % NKV) * F16_BUF + F16_TILE;
            const uint64_t vdesc[4] = {smem_desc_sw128(vbuf), smem_desc_sw128(vbuf + 2048),
                                       smem_desc_sw128(vbuf + 4096), smem_desc_sw128(vbuf + 6144)};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                if (!wait_warp(BAR(BAR_P_FULL + 2 * w + (k & 1)), (k >> 1) & 1, abort_flag)) return false;
                if (first && seg >= 1 && !wait_warp(BAR(BAR_O_FREE + w), (seg - 1) & 1, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t pa = tmem + TM_S + 128u * w + 64u * (k & 1);
                const uint32_t av[4] = {pa, pa + 8u, pa + 16u, pa + 24u};
                tc_mma_ts4(tmem + TM_O + 64u * w, av, vdesc, ID_O, first ? 0u : 1u);
            }
            tc_commit(BAR(BAR_KV_FREE + k % NKV));
            return true;
        };
        int ct = t0, cb = find_req(t0);
        int seg_b = -1, seg = -1;
        bool prev_first = false;
        int prev_seg = -1;
        bool ok = true;
        int i = 0;
        for (; ct < t1; ++i) {
            const bool first = cb != seg_b;
            if (first) {
                seg_b = cb;
                ++seg;
            }
            // At an item's first tile the previous item's last P.V goes first: its
            // softmax warpgroups read O out after it and only then write the new
            // item's Q, which the S MMAs below wait for.
            if (first && i > 0 && !issue_pv(i - 1, prev_first, prev_seg)) {
                ok = false;
                break;
            }
            if (!wait_warp(BAR(BAR_KV_READY + i % NKV), (i / NKV) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t kbuf = f16_base + (i % NKV) * F16_BUF;
            const uint64_t kdesc[4] = {smem_desc_sw128(kbuf), smem_desc_sw128(kbuf + 32),
                                       smem_desc_sw128(kbuf + 64), smem_desc_sw128(kbuf + 96)};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                if (first) {  // the item's Q_w, written by its softmax warpgroup
                    if (!wait_warp(BAR(BAR_Q_READY + w), seg & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                const uint32_t sd = tmem + TM_S + 128u * w + 64u * (i & 1);
                const uint32_t qa = tmem + TM_Q + 32u * w;
                const uint32_t aq[4] = {qa, qa + 8u, qa + 16u, qa + 24u};
                tc_mma_ts4(sd, aq, kdesc, ID_S, 0u);
                tc_commit(BAR(BAR_S_FULL + 2 * w + (i & 1)));
            }
            if (!ok) break;
            // within an item, P.V of the previous tile runs behind this tile's S
            if (!first && i > 0 && !issue_pv(i - 1, prev_first, prev_seg)) {
                ok = false;
                break;
            }
            prev_first = first;
            prev_seg = seg;
            advance(ct, cb);
        }
        if (ok && i > 0) issue_pv(i - 1, prev_first, prev_seg);
        // every MMA this warp issued is done before the tensor memory is freed
        tc_commit(BAR(BAR_MMA_DONE));
        const bool done = wait_bounded(BAR(BAR_MMA_DONE), 0, abort_flag, false, TEARDOWN_LIMIT_NS);
        __syncwarp();
        (void)done;
    } else {
        // =================== softmax: warpgroup w, one thread per row of tile w ===================
        const int w = warp >> 2;
        const int r = tid - SM_THREADS * w;
        const int jt = 16 * w + (r >> 3), hh = r & 7;  // token in the chunk, head of the KV head
        const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const uint32_t s_base = tmem + TM_S + 128u * w + lane_base;
        const uint32_t o_base = tmem + TM_O + 64u * w + lane_base;
        const uint32_t q_row = tmem + TM_Q + 32u * w + lane_base;
        bool prep_done = false;
        int ct = t0, cb = find_req(t0);
        int seg_b = -1, seg_t1 = 0, k0 = 0;  // current item, end of its tiles here, tile key
        float m_run = -INFINITY, l_run = 0.f;
        int lo_j = INT_MAX, hi_j = -1;
        int seg_len = 0;  // tokens of the current item
        for (int i = 0; ct < t1; ++i) {
            const bool seg_start = cb != seg_b;
            if (seg_start) {
                seg_b = cb;
                seg_t1 = min(t1, tpre[cb + 1]);
                k0 = tile_k0(ct, cb);
                m_run = -INFINITY;
                l_run = 0.f;
                const ItemRef it = item_ref<true>(p, cb);
                seg_len = it.len;
                // this row of Q_w (the S MMAs of the previous item, which read
                // Q_w, are done: their S was consumed above)
                if (!prep_done) {
                    pdl_wait_primary();  // q comes from the prep kernel
                    prep_done = true;
                }
                uint32_t q[32];
                if (jt < it.len) {
                    const int pos = static_cast<int>(p.positions[static_cast<size_t>(it.t0) + jt]);
                    hi_j = pos;
                    lo_j = p.window > 0 ? max(0, pos - p.window + 1) : 0;
                    const uint4* src = reinterpret_cast<const uint4*>(
                        p.q_ws + ((static_cast<size_t>(it.t0) + jt) * HQ + it.grp * GRP + hh) * HD);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v = src[c];
                        q[4 * c] = v.x;
                        q[4 * c + 1] = v.y;
                        q[4 * c + 2] = v.z;
                        q[4 * c + 3] = v.w;
                    }
                } else {
                    lo_j = INT_MAX;
                    hi_j = -1;
#pragma unroll
                    for (int c = 0; c < 32; ++c) q[c] = 0u;
                }
                tc_st32(q_row, q);
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(BAR_Q_READY + w));
            } else {
                k0 += TK;
            }
            const bool seg_end = ct + 1 >= seg_t1;

            if (!wait_warp(BAR(BAR_S_FULL + 2 * w + (i & 1)), (i >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t sbuf = s_base + 64u * (i & 1);
            uint32_t sr[64];
            tc_ld32(sbuf, sr);
            tc_ld32(sbuf + 32u, sr + 32);
            tc_wait_ld();
            float s[64];
            const int cmin = lo_j == INT_MAX ? TK : lo_j - k0;
            const int cmax = hi_j - k0;
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (cmin <= 0 && cmax >= TK - 1) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    s[c] = __uint_as_float(sr[c]);
                    m4[c & 3] = fmaxf(m4[c & 3], s[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    s[c] = (c < cmin || c > cmax) ? -INFINITY : __uint_as_float(sr[c]);
                    m4[c & 3] = fmaxf(m4[c & 3], s[c]);
                }
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // lazy rescale: O (in tensor memory) is corrected only when the max grows a lot
            const float m_new = fmaxf(m_run, mx);
            bool corr = false;
            if (m_new > m_run) {
                if (m_run == -INFINITY || seg_start || (m_new - m_run) * C2 <= RESCALE_LOG2) {
                    if (m_run == -INFINITY || seg_start) m_run = m_new;
                } else {
                    corr = true;
                }
            }
            if (__any_sync(0xffffffffu, corr)) {
                // the P.V of tile i - 1 (same item) must be done before O is touched
                if (!wait_warp(BAR(BAR_KV_FREE + (i - 1) % NKV), ((i - 1) / NKV) & 1, abort_flag)) break;
                tc_fence_after();
                const float alpha = corr ? fast_exp2((m_run - m_new) * C2) : 1.f;
                uint32_t o[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tc_ld32(o_base + 32u * half, o);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tc_st32(o_base + 32u * half, o);
                }
                tc_wait_st();
                if (corr) {
                    l_run *= alpha;
                    m_run = m_new;
                }
            }
            const float mc = m_run == -INFINITY ? 0.f : m_run * C2;
            uint32_t pk[32];
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
            // every POLY_EVERY-th pair's second weight on the FMA pipe, the
            // rest on the MUFU unit, so the two run side by side
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float p0 = fast_exp2(fmaf(s[2 * c], C2, -mc));
                const float x1 = fmaf(s[2 * c + 1], C2, -mc);
                const float p1 = c % POLY_EVERY == 0 ? exp2_poly(x1) : fast_exp2(x1);
                l4[c & 3] += p0 + p1;
                pk[c] = pack_f16x2(p0, p1);
            }
            l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            tc_st32(sbuf, pk);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(BAR_P_FULL + 2 * w + (i & 1)));

            if (seg_end) {
                if (!wait_warp(BAR(BAR_KV_FREE + i % NKV), (i / NKV) & 1, abort_flag)) break;
                tc_fence_after();
                const size_t slot = static_cast<size_t>(blockIdx.x) + cb;
                const size_t base = (slot * p.lt + jt) * p.hp + hh;
                uint32_t o[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tc_ld32(o_base + 32u * half, o);
                    tc_wait_ld();
                    if (jt < seg_len) {
                        float4* dst = reinterpret_cast<float4*>(p.part_o + base * HD + 32 * half);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                                 __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
                    }
                }
                if (jt < seg_len) {
                    p.part_ml[base * 2 + 0] = m_run * C2;
                    p.part_ml[base * 2 + 1] = l_run;
                }
                tc_fence_before();
                mbar_arrive(BAR(BAR_O_FREE + w));
            }
            ++ct;
            if (seg_end)
                while (cb < B - 1 && ct >= tpre[cb + 1]) ++cb;
        }
    }

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tc_dealloc(tmem, TM_COLS);
    }
    if (tid == 0 && *abort_flag) {
        pdl_wait_primary();  // the step's first kernel has cleared the status word
        atomicOr(p.status, STATUS_ATTN_WAIT);
    }
    pdl_launch_dependents();
}

}  // namespace gad
