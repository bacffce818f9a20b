// gad_kernels.cuh - the step's shared definitions (head groups, StepParams,
// the tile list) and its single-token attention kernel.
//
//   decode_kernel   persistent split-KV flash decode over the paged FP8 cache:
//                   cp.async gathers into a swizzled shared-memory ring, tensor-
//                   core QK^T and PV (m16n8k16 fp16, fp32 accumulate) with the
//                   query heads of one KV head packed into the MMA's N side,
//                   online softmax, one (o, max, sum) partial per CTA segment.
//   (prep_kernel, per token QK-norm, RoPE and the E4M3 cache append, is in
//   gad_prep.cuh; the combine kernels, which merge the partials and apply the
//   gated output norm, are in gad_combine.cuh)
//
// Method: task page "Gated attention decode (muse_attention_decode)", section
// "What to compute"; shapes from its section "Shapes".
#pragma once

#include <cfloat>
#include <climits>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "gad_ptx.cuh"
#include "gad_tc.cuh"

namespace gad {

// Head groups.  The kernels work on groups of 16 query heads over 2 KV heads
// (query head h of a group reads its KV head h / 8).  The page's "heads tp8"
// shapes are one group; a step with ngrp groups (16 ngrp query heads, 2 ngrp
// KV heads, e.g. 8 groups for "heads dp") is ngrp independent problems that
// share positions, pages and cache rows.  Columns of a qkv row, for group c:
//   q    c * 1024 + 64 h                    (section of 1024 ngrp columns)
//   k    1024 ngrp + 128 c + 64 g           (section of 128 ngrp)
//   v    1152 ngrp + 128 c + 64 g           (section of 128 ngrp)
//   gate 1280 ngrp + 1024 c + 64 h          (section of 1024 ngrp)
// a cache row holds 128 ngrp bytes (group c at byte 128 c), and an output row
// 1024 ngrp values (group c at 1024 c).
constexpr int HQ = 16;         // query heads of a group
constexpr int HKV = 2;         // key/value heads of a group
constexpr int HD = 64;         // head dim
constexpr int GRP = HQ / HKV;  // query heads per KV head (8)
constexpr int QKV_COLS = 2304; // qkv columns per group
constexpr int K_OFF = 1024, V_OFF = 1152, G_OFF = 1280;  // section starts per group
constexpr int OUT_COLS = 1024; // output columns per group
constexpr int ROWB = 128;                   // cache bytes per row and group: 2 KV heads x 64 codes
constexpr int TILE = 64;                    // keys per pipeline stage
constexpr int STAGE_BYTES = 2 * TILE * ROWB;  // K tile then V tile: 16 KB
constexpr int DEC_THREADS = 256;
constexpr int PREP_THREADS = (HQ + HKV) * 32;

struct StepParams {
    const __nv_bfloat16* qkv;
    const int64_t* positions;
    const int32_t* page_table;
    const int64_t* cache_loc;
    uint8_t* k_cache;
    uint8_t* v_cache;
    const float* k_scale;
    const float* v_scale;
    __nv_bfloat16* out;
    int B, L, max_pages, window, use_rope;
    int ngrp;        // head groups (16 query + 2 KV heads each)
    int chunk;       // tokens per item chunk (CHUNK, or PF_CHUNK for prefill_tc_kernel)
    int nchunk;      // token chunks per request: ceil(L / chunk)
    int nsub;        // items per chunk: head groups, or KV heads for prefill_tc_kernel
    int hp;          // query heads per partial row block (16, or 8 for prefill_tc_kernel)
    int NB;          // items of the tile list: B * nchunk * nsub (see ItemRef)
    int64_t num_rows;
    // workspace views
    __half* q_ws;    // [T][ngrp][16][64]  normalised (rotated) queries
    float* part_o;   // [slots][lt][16][64]  un-normalised partial outputs (slot = CTA + item)
    float* part_ml;  // [slots][lt][16][2]   (running max in log2 units, sum)
    int* meta;       // see META_*: tile count, tiles per CTA, tile prefix over items
    int* status;     // the step's status word (STATUS_* bits), at offset 0 of the workspace
    double inv_freq[HD / 2];  // RoPE: 10000^(-2i/64) for pair i, computed on the host
    int lt;          // token capacity of one partial slot (1 or 8)
    int tl;          // partials per (CTA, request) and KV-head group
};

// Items of the tile list.  Item i = (request, token chunk, sub) with
// i = (request * nchunk + chunk) * nsub + sub: a chunk is up to p.chunk
// consecutive tokens of one request (a whole decode token or verify block,
// or a slice of a longer prefill block), and its key range is the union of
// its tokens' ranges.  sub is the head group for decode_kernel and
// verify_tc_kernel, the KV head for prefill_tc_kernel.  The MULTI = false
// instantiations serve steps with one item per request, where item = request.
constexpr int CHUNK = 8;      // tokens per item: decode and verify kernels
constexpr int PF_CHUNK = 32;  // tokens per item: prefill_tc_kernel
struct ItemRef {
    int req;   // request
    int grp;   // sub: head group, or KV head (prefill_tc_kernel)
    int t0;    // first token (global index b * L + j)
    int len;   // tokens in the chunk
};
template <bool MULTI>
__device__ __forceinline__ ItemRef item_ref(const StepParams& p, int i) {
    if (!MULTI) return ItemRef{i, 0, i * p.L, p.L};
    const int sub = i % p.nsub, rc = i / p.nsub;
    const int chunk = rc % p.nchunk, req = rc / p.nchunk;
    const int j0 = chunk * p.chunk;
    return ItemRef{req, sub, req * p.L + j0, min(p.chunk, p.L - j0)};
}

// Layout of StepParams::meta (ints).
constexpr int META_TOTAL = 0;    // tiles in the step
constexpr int META_PER = 1;      // tiles per CTA
constexpr int META_PREFIX = 3;   // [NB + 1] tile prefix over list items
constexpr int META_INTS = 4;     // + NB

// Bits of the step's status word.  The step's first kernel clears the word;
// a kernel whose bounded wait gave up sets its bit at the end, after waiting
// for the kernel before it (so the clear is always ordered first).
constexpr int STATUS_ATTN_WAIT = 1;   // an attention kernel's wait timed out
constexpr int STATUS_OPROJ_WAIT = 2;  // the output projection's wait timed out

// ---------------------------------------------------------------------------
// Kernel 2: split-KV decode.
//
// Work split.  Request b attends keys [lo_b, hi_b] (the union of its tokens'
// ranges).  Its keys fall into 64-key tiles aligned to absolute key index
// (so a 64-key page is exactly one tile).  All requests' tiles form one list;
// CTA c takes tiles [c*per, (c+1)*per) of it, crossing request boundaries,
// and writes one partial per (CTA, request) it touches into slot c + b
// (unique, since both c and b only grow along the list).
//
// Shared-memory tile layout.  A stage holds 64 rows of K then 64 rows of V,
// 128 bytes per row (both KV heads), 16-byte chunk j of row r stored at chunk
// j ^ (r & 7) (the 128-byte swizzle).  The MMA's logical key l in a 16-key
// group lives in row kappa(l) of that group; kappa is chosen so that both the
// QK^T operand loads (16 bytes per lane) and the PV operand loads (8 bytes per
// lane) are free of bank conflicts under that swizzle.
//
// MMA mapping (m16n8k16, transposed so the 8 query heads of a KV head fill N):
//   S^T[key][head] = K[key][:] . Q[head][:]        A = K (fp16 from E4M3), B = Q
//   O^T[dim][head] += V^T[dim][key] . P^T[key][head]  A = V^T, B = P^T
// Each lane holds 16 contiguous K bytes of a row (dims permuted across k-steps
// identically for K and Q), and 8 contiguous V dims; P^T's B fragment comes
// from S^T's accumulator by one movmatrix transpose per 8x8 block.
//
// Warps: 8 = 2 KV heads x RG row groups (tokens) x KG key groups.  Each warp
// runs its own online softmax over its keys; key groups are merged in shared
// memory at the end of each segment.
// ---------------------------------------------------------------------------
// Per-item key ranges [lo_i, hi_i] (union over the item's request's tokens),
// the first key this step writes (rnew_i), the prefix of TK-key tile counts
// over the list items (tiles aligned to multiples of TK), and this CTA's share
// of the tile list [t0, t1).  Item i is request i / ngrp and head group
// i % ngrp, so a request's groups are adjacent in the list and the CTAs that
// share its pages run at about the same time.  Every thread of the block must
// call it.  CTA 0 also writes the list to the workspace for the combine kernel.
template <int TK, bool MULTI>
__device__ __forceinline__ void build_tile_list(const StepParams& p, int* tpre, int* rlo, int* rhi,
                                                int* rnew, int nthreads, int& total, int& per,
                                                int& t0, int& t1) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = MULTI ? p.NB : p.B;
    for (int b = tid; b < B; b += nthreads) {
        const ItemRef it = item_ref<MULTI>(p, b);
        int lo = INT_MAX, hi = -1, first = INT_MAX;
        for (int j = 0; j < it.len; ++j) {
            const int pos = static_cast<int>(p.positions[static_cast<size_t>(it.t0) + j]);
            const int l = p.window > 0 ? max(0, pos - p.window + 1) : 0;
            lo = min(lo, l);
            hi = max(hi, pos);
            first = min(first, pos);
        }
        // Keys at or above the request's first position are written by this
        // step (by the prep kernel, which may still be running), including the
        // keys of the request's earlier chunks.
        if (MULTI) first = min(first, static_cast<int>(p.positions[static_cast<size_t>(it.req) * p.L]));
        rlo[b] = lo;
        rhi[b] = hi;
        rnew[b] = first;
        tpre[b + 1] = (hi >= lo && hi >= 0) ? (hi / TK - lo / TK + 1) : 0;
    }
    if (tid == 0) tpre[0] = 0;
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 1; base <= B; base += 32) {
            const int i = base + lane;
            int v = i <= B ? tpre[i] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (i <= B) tpre[i] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();
    total = tpre[B];
    per = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
    t0 = static_cast<int>(blockIdx.x) * per;
    t1 = min(t0 + per, total);
    if (blockIdx.x == 0) {
        for (int i = tid; i <= B; i += nthreads) p.meta[META_PREFIX + i] = tpre[i];
        if (tid == 0) {
            p.meta[META_TOTAL] = total;
            p.meta[META_PER] = per;
        }
    }
}

template <int LT, int KG, int NS, int TK, bool MERGE>
struct DecodeCfg {
    static constexpr int WARPS = DEC_THREADS / 32;
    static constexpr int RG = WARPS / (HKV * KG);
    static constexpr int NT = LT / RG;              // tokens per warp (MMA N tiles)
    static constexpr int MT = (TK / 16) / KG;       // 16-key groups per warp per tile
    static constexpr int STAGE = 2 * TK * ROWB;     // K tile then V tile
    static constexpr int IDX_SLOTS = 2 * NS;
    static constexpr int MERGE_WARPS = MERGE ? (KG - 1) * HKV * RG : 0;
    static constexpr int MERGE_FLOATS_PER_WARP = NT * 32 * 20;
    // partials per (CTA, request): one after the in-CTA merge, else one per key group
    static constexpr int PARTS = MERGE ? 1 : KG;
    static constexpr size_t KV_BYTES = static_cast<size_t>(NS) * STAGE;
    static constexpr size_t IDX_BYTES = static_cast<size_t>(IDX_SLOTS) * TK * 4;
    static constexpr size_t MERGE_BYTES =
        static_cast<size_t>(MERGE_WARPS) * MERGE_FLOATS_PER_WARP * 4;
    // page size 64: one mbarrier per stage (the TMA page loads' bytes) and the
    // abort flag
    static constexpr size_t CTRL_BYTES = 64;
    static_assert(NS * 8 + 8 <= static_cast<int>(CTRL_BYTES), "control block");
    // + 1024 so the stages can start on a 1024-byte boundary (the 128-byte
    // swizzle of the TMA page loads is anchored there)
    static size_t smem_bytes(int B) {
        return 1024 + KV_BYTES + IDX_BYTES + MERGE_BYTES + CTRL_BYTES + static_cast<size_t>(4 * B + 1) * 4;
    }
    static_assert(RG >= 1 && RG * HKV * KG == WARPS, "warp split");
    static_assert(NT * RG == LT && MT * KG == TK / 16, "tile split");
    static_assert(TK % 64 == 0 && TK <= DEC_THREADS, "tile size");
};

// Row (within a 16-key group) holding the MMA's logical key l.
__device__ __forceinline__ int kappa(int l) {
    const int x = l & 7;
    const int s = ((((x & 1) << 2) ^ (((x >> 1) & 3) << 1)) | ((x >> 2) & 1));
    return (l & 8) | s;
}

// MULTI: more than one head group (the one-group instantiation keeps the
// list item equal to the request, with no index arithmetic for groups).
// Page size 64: a stage's pages arrive by TMA tile loads (kmap, vmap: the K and
// V caches as 2D tensors of 128 ngrp-byte rows, one 64-row page x 128 bytes a
// tile, 128-byte swizzle: the layout the page-size-1 gathers write), issued
// by thread 0 and waited for on the stage's mbarrier.
template <int LT, int PS, int KG, int NS, int MINB, int TK, bool MERGE, bool MULTI>
__global__ void __launch_bounds__(DEC_THREADS, MINB)
    decode_kernel(const StepParams p, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap) {
    using C = DecodeCfg<LT, KG, NS, TK, MERGE>;
    constexpr int NT = C::NT, MT = C::MT, RG = C::RG;
    constexpr bool TMA = PS == 64;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* kv_smem = smem;
    int* idx_smem = reinterpret_cast<int*>(smem + C::KV_BYTES);
    float* merge_smem = reinterpret_cast<float*>(smem + C::KV_BYTES + C::IDX_BYTES);
    uint8_t* ctrl = smem + C::KV_BYTES + C::IDX_BYTES + C::MERGE_BYTES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + NS * 8);
    int* tpre = reinterpret_cast<int*>(ctrl + C::CTRL_BYTES);
    int* rlo = tpre + p.NB + 1;
    int* rhi = rlo + p.NB;
    int* rnew = rhi + p.NB;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int g = warp % HKV;
    const int rg = (warp / HKV) % RG;
    const int kg = warp / (HKV * RG);
    // B counts list items (request, head group); b below is an item index.
    const int B = MULTI ? p.NB : p.B, ng = MULTI ? p.ngrp : 1;
    const size_t row_pitch = static_cast<size_t>(ROWB) * ng;  // cache bytes per row

    // ---- request key ranges and the tile list (reads inputs only) ----
    int total, per, t0, t1;
    build_tile_list<TK, MULTI>(p, tpre, rlo, rhi, rnew, DEC_THREADS, total, per, t0, t1);
    if (t0 >= t1) return;
    const uint32_t bar0 = smem_addr(ctrl);
    auto STAGE_BAR = [&](int st) { return bar0 + 8u * static_cast<uint32_t>(st); };
    if (TMA) {
        if (tid == 0) {
            for (int st = 0; st < NS; ++st) mbar_init(STAGE_BAR(st), 1);
            *abort_flag = 0;
            mbar_fence_init();
        }
        __syncthreads();
    }
    // The normalised q and this step's new cache rows come from the prep kernel,
    // which may still be running (programmatic dependent launch): wait for it
    // only before the first q load or the first gather of a tile holding new
    // keys, so the tile list and the first gathers overlap it.  The condition is
    // the same for every thread of the CTA.
    bool prep_done = false;
    auto ensure_prep = [&]() {
        if (!prep_done) {
            pdl_wait_primary();
            prep_done = true;
        }
    };

    const float C2 = __ldg(p.k_scale) * 0.125f * 1.4426950408889634f;  // raw score -> log2 units

    // ---- tile cursors ----
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

    // ---- async loads ----
    auto issue_idx = [&](int tau, int b) {
        if (tau >= t1) return;
        const int k0 = tile_k0(tau, b);
        int* dst = idx_smem + ((tau - t0) % C::IDX_SLOTS) * TK;
        const int32_t* pt = p.page_table + static_cast<size_t>(item_ref<MULTI>(p, b).req) * p.max_pages;
        if (PS == 1) {
            if (tid < TK) {
                const int k = k0 + tid;
                if (k >= rlo[b] && k <= rhi[b] && k < p.max_pages) cp_async4(smem_addr(dst + tid), pt + k);
                else dst[tid] = -1;
            }
        } else {
            if (tid < TK / PS) {  // the tile's pages
                const int pg = k0 / PS + tid;
                if (pg < p.max_pages) cp_async4(smem_addr(dst + tid), pt + pg);
                else dst[tid] = -1;
            }
        }
    };
    int n_issued = 0;  // tiles whose loads were issued (the same count in every thread)
    auto issue_kv = [&](int tau, int b) {
        if (tau >= t1) return;
        const int k0 = tile_k0(tau, b);
        if (k0 + TK - 1 >= rnew[b]) ensure_prep();
        const int* ix = idx_smem + ((tau - t0) % C::IDX_SLOTS) * TK;
        const uint32_t base = smem_addr(kv_smem + ((tau - t0) % NS) * C::STAGE);
        const int lo = rlo[b], hi = rhi[b];
        const size_t gofs = static_cast<size_t>(item_ref<MULTI>(p, b).grp) * ROWB;
        ++n_issued;
        if constexpr (TMA) {
            // the tile's TK / 64 pages, K and V: one TMA tile load each; a page
            // index past the table (-1) or rows past the cache fall outside the
            // tensor and read as zeros
            if (tid == 0) {
                fence_proxy_async_smem();  // the zeroed rows of this stage's last tile come first
                const uint32_t bar = STAGE_BAR((tau - t0) % NS);
                mbar_arrive_expect_tx(bar, C::STAGE);
#pragma unroll
                for (int pq = 0; pq < TK / PS; ++pq) {
                    const int pg = ix[pq];
                    const int y = pg >= 0 ? pg * PS : -PS;
                    tma_load_2d(base + pq * PS * ROWB, &kmap, static_cast<int>(gofs), y, bar);
                    tma_load_2d(base + TK * ROWB + pq * PS * ROWB, &vmap, static_cast<int>(gofs), y, bar);
                }
            }
        } else {
            static_assert(PS == 1, "page size 64 reads whole pages by TMA");
#pragma unroll
            for (int i = 0; i < TK / 32; ++i) {
                const int r = (tid >> 3) + 32 * i;  // tile row
                const int j = tid & 7;              // 16-byte chunk
                const int k = k0 + r;
                const int64_t crow = ix[r];
                const bool ok = k >= lo && k <= hi && crow >= 0 && crow < p.num_rows;
                const size_t off = ok ? static_cast<size_t>(crow) * row_pitch + gofs + j * 16 : 0;
                const uint32_t d = base + r * ROWB + ((j ^ (r & 7)) << 4);
                cp_async16(d, p.k_cache + off, ok ? 16 : 0);
                cp_async16(d + TK * ROWB, p.v_cache + off, ok ? 16 : 0);
            }
        }
    };

    // ---- per-warp state ----
    float o_acc[NT][4][4];
    float m_run[NT][2], l_run[NT][2];
    uint32_t qf[NT][8];
    int tok_lo[NT], tok_hi[NT];
    int req_lo_max = 0, req_hi_min = -1;
    int cur_len = 0;  // tokens of the current item

    const int krow = kappa(gid);             // QK^T: rows krow, krow + 8 of each group
    const int vrow0 = kappa(2 * tig), vrow1 = kappa(2 * tig + 1);  // PV: + 0 and + 8

    auto begin_request = [&](int b) {
        ensure_prep();
        const ItemRef it = item_ref<MULTI>(p, b);
        cur_len = it.len;
        req_lo_max = 0;
        req_hi_min = INT_MAX;
        for (int j = 0; j < it.len; ++j) {
            const int pos = static_cast<int>(p.positions[static_cast<size_t>(it.t0) + j]);
            const int l = p.window > 0 ? max(0, pos - p.window + 1) : 0;
            req_lo_max = max(req_lo_max, l);
            req_hi_min = min(req_hi_min, pos);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int j = rg * NT + nt;
            if (j < it.len) {
                const size_t t = static_cast<size_t>(it.t0) + j;
                const int pos = static_cast<int>(p.positions[t]);
                tok_hi[nt] = pos;
                tok_lo[nt] = p.window > 0 ? max(0, pos - p.window + 1) : 0;
                const uint4* q = reinterpret_cast<const uint4*>(
                    p.q_ws + ((t * ng + it.grp) * HQ + g * GRP + gid) * HD + 16 * tig);
                const uint4 a = q[0], c = q[1];
                qf[nt][0] = a.x; qf[nt][1] = a.y; qf[nt][2] = a.z; qf[nt][3] = a.w;
                qf[nt][4] = c.x; qf[nt][5] = c.y; qf[nt][6] = c.z; qf[nt][7] = c.w;
            } else {
                tok_lo[nt] = INT_MAX;
                tok_hi[nt] = -1;
#pragma unroll
                for (int i = 0; i < 8; ++i) qf[nt][i] = 0u;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                m_run[nt][e] = -INFINITY;
                l_run[nt][e] = 0.f;
            }
#pragma unroll
            for (int dt = 0; dt < 4; ++dt)
#pragma unroll
                for (int c = 0; c < 4; ++c) o_acc[nt][dt][c] = 0.f;
        }
    };

    auto compute_tile = [&](int slot, int k0) {
        const uint32_t kbase = smem_addr(kv_smem + slot * C::STAGE);
        const uint32_t vbase = kbase + TK * ROWB;
        const bool need_mask = !(k0 >= req_lo_max && k0 + TK - 1 <= req_hi_min);
        float s[MT][NT][4];
        // S^T = K . Q^T
#pragma unroll
        for (int i = 0; i < MT; ++i) {
            const int ra = (kg * MT + i) * 16 + krow;
            const uint32_t chunk = static_cast<uint32_t>(((4 * g + tig) ^ (ra & 7)) << 4);
            const uint4 ka = lds128(kbase + ra * ROWB + chunk);
            const uint4 kb = lds128(kbase + (ra + 8) * ROWB + chunk);
            const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w};
            const uint32_t kbw[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[i][nt][c] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2(kaw[ks]);
                a[1] = e4m3x2_to_f16x2(kbw[ks]);
                a[2] = e4m3x2_to_f16x2(kaw[ks] >> 16);
                a[3] = e4m3x2_to_f16x2(kbw[ks] >> 16);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_16816(s[i][nt], a, qf[nt][2 * ks], qf[nt][2 * ks + 1]);
            }
        }
        if (need_mask) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int key_a = k0 + (kg * MT + i) * 16 + krow;
                const int key_b = key_a + 8;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (key_a < tok_lo[nt] || key_a > tok_hi[nt]) s[i][nt][0] = s[i][nt][1] = -INFINITY;
                    if (key_b < tok_lo[nt] || key_b > tok_hi[nt]) s[i][nt][2] = s[i][nt][3] = -INFINITY;
                }
            }
        }
        // online softmax (per token, per head 2*tig + e)
        uint32_t pf[MT][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < MT; ++i) mx = fmaxf(mx, fmaxf(s[i][nt][e], s[i][nt][2 + e]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[nt][e], mx);
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = fast_exp2((m_run[nt][e] - m_use) * C2);
                m_run[nt][e] = m_new;
                float lsum = l_run[nt][e] * alpha;
#pragma unroll
                for (int dt = 0; dt < 4; ++dt) {
                    o_acc[nt][dt][e] *= alpha;
                    o_acc[nt][dt][2 + e] *= alpha;
                }
                const float mc = m_use * C2;
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    const float p0 = fast_exp2(fmaf(s[i][nt][e], C2, -mc));
                    const float p1 = fast_exp2(fmaf(s[i][nt][2 + e], C2, -mc));
                    s[i][nt][e] = p0;
                    s[i][nt][2 + e] = p1;
                    lsum += p0 + p1;
                }
                l_run[nt][e] = lsum;
            }
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                pf[i][nt][0] = movmatrix_t(pack_f16x2(s[i][nt][0], s[i][nt][1]));
                pf[i][nt][1] = movmatrix_t(pack_f16x2(s[i][nt][2], s[i][nt][3]));
            }
        }
        // O^T += V^T . P^T
#pragma unroll
        for (int i = 0; i < MT; ++i) {
            const int gb = (kg * MT + i) * 16;
            const int r0 = gb + vrow0, r1 = gb + vrow1;
            const int cpos = 4 * g + (gid >> 1);
            const uint32_t sub = static_cast<uint32_t>((gid & 1) * 8);
            const uint2 x0 = lds64(vbase + r0 * ROWB + ((cpos ^ (r0 & 7)) << 4) + sub);
            const uint2 x1 = lds64(vbase + r1 * ROWB + ((cpos ^ (r1 & 7)) << 4) + sub);
            const uint2 x2 = lds64(vbase + (r0 + 8) * ROWB + ((cpos ^ (r0 & 7)) << 4) + sub);
            const uint2 x3 = lds64(vbase + (r1 + 8) * ROWB + ((cpos ^ (r1 & 7)) << 4) + sub);
#pragma unroll
            for (int dt = 0; dt < 4; ++dt) {
                const uint32_t w0 = dt < 2 ? x0.x : x0.y, w1 = dt < 2 ? x1.x : x1.y;
                const uint32_t w2 = dt < 2 ? x2.x : x2.y, w3 = dt < 2 ? x3.x : x3.y;
                const uint32_t sel = (dt & 1) ? 0x7362u : 0x5140u;
                const uint32_t p01 = __byte_perm(w0, w1, sel);
                const uint32_t p23 = __byte_perm(w2, w3, sel);
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2(p01);
                a[1] = e4m3x2_to_f16x2(p01 >> 16);
                a[2] = e4m3x2_to_f16x2(p23);
                a[3] = e4m3x2_to_f16x2(p23 >> 16);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_16816(o_acc[nt][dt], a, pf[i][nt][0], pf[i][nt][1]);
            }
        }
    };

    auto flush = [&](int b) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float l = l_run[nt][e];
                l += __shfl_xor_sync(0xffffffffu, l, 4);
                l += __shfl_xor_sync(0xffffffffu, l, 8);
                l += __shfl_xor_sync(0xffffffffu, l, 16);
                l_run[nt][e] = l;
            }
        if (MERGE && KG > 1) {
            if (kg > 0) {
                float* buf = merge_smem +
                             static_cast<size_t>(((kg - 1) * HKV * RG + g * RG + rg) * NT) * 640;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float* d = buf + (nt * 32 + lane) * 20;
#pragma unroll
                    for (int dt = 0; dt < 4; ++dt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) d[dt * 4 + c] = o_acc[nt][dt][c];
                    d[16] = m_run[nt][0];
                    d[17] = m_run[nt][1];
                    d[18] = l_run[nt][0];
                    d[19] = l_run[nt][1];
                }
            }
            __syncthreads();
            if (kg == 0) {
                for (int k = 1; k < KG; ++k) {
                    const float* buf = merge_smem +
                                       static_cast<size_t>(((k - 1) * HKV * RG + g * RG + rg) * NT) * 640;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const float* d = buf + (nt * 32 + lane) * 20;
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float mo = d[16 + e], lo = d[18 + e];
                            const float M = fmaxf(m_run[nt][e], mo);
                            if (M == -INFINITY) continue;
                            const float a = fast_exp2((m_run[nt][e] - M) * C2);
                            const float ao = fast_exp2((mo - M) * C2);
                            l_run[nt][e] = a * l_run[nt][e] + ao * lo;
                            m_run[nt][e] = M;
#pragma unroll
                            for (int dt = 0; dt < 4; ++dt) {
                                o_acc[nt][dt][e] = a * o_acc[nt][dt][e] + ao * d[dt * 4 + e];
                                o_acc[nt][dt][2 + e] = a * o_acc[nt][dt][2 + e] + ao * d[dt * 4 + 2 + e];
                            }
                        }
                    }
                }
            }
            __syncthreads();
        }
        if (!MERGE || kg == 0) {
            const size_t slot = (static_cast<size_t>(blockIdx.x) + b) * C::PARTS + (MERGE ? 0 : kg);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int j = rg * NT + nt;
                if (j >= cur_len) continue;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int h = g * GRP + 2 * tig + e;
                    const size_t base = (slot * p.lt + j) * HQ + h;
                    float4* dst = reinterpret_cast<float4*>(p.part_o + base * HD + 8 * gid);
                    dst[0] = make_float4(o_acc[nt][0][e], o_acc[nt][0][2 + e], o_acc[nt][1][e],
                                         o_acc[nt][1][2 + e]);
                    dst[1] = make_float4(o_acc[nt][2][e], o_acc[nt][2][2 + e], o_acc[nt][3][e],
                                         o_acc[nt][3][2 + e]);
                    if (gid == 0) {
                        p.part_ml[base * 2 + 0] = m_run[nt][e] * C2;
                        p.part_ml[base * 2 + 1] = l_run[nt][e];
                    }
                }
            }
        }
    };

    // ---- pipeline ----
    int xt = t0, xb = find_req(t0);  // idx issue cursor
    int kt = t0, kb = xb;            // kv issue cursor
    int ct = t0, cb = xb;            // compute cursor
    for (int d = 0; d < NS - 1; ++d) {
        issue_idx(xt, xb);
        advance(xt, xb);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    for (int d = 0; d < NS - 1; ++d) {
        issue_kv(kt, kb);
        advance(kt, kb);
        issue_idx(xt, xb);
        advance(xt, xb);
        cp_async_commit();
    }
    int cur_b = -1;
    int i = 0;
    for (; ct < t1; ++i) {
        cp_async_wait<NS - 2>();
        if constexpr (TMA) {
            // the stage's pages landed; keys of the tile outside the item's range
            // (page slots not yet written, or before a window) become zeros, as
            // the page-size-1 gathers zero-fill them: thread (row, half) clears
            // its half of the K and V rows
            bool bad = !wait_bounded(STAGE_BAR(i % NS), (i / NS) & 1, abort_flag);
            const int k0 = tile_k0(ct, cb);
            const int r = tid >> 1;
            if (!bad && (k0 + r < rlo[cb] || k0 + r > rhi[cb])) {
                const uint32_t row = smem_addr(kv_smem + (i % NS) * C::STAGE) + r * ROWB + (tid & 1) * 64;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sts128(row + 16 * q, make_uint4(0u, 0u, 0u, 0u));
                    sts128(row + TK * ROWB + 16 * q, make_uint4(0u, 0u, 0u, 0u));
                }
                fence_proxy_async_smem();
            }
            if (bar_red_or(0, DEC_THREADS, bad)) break;
        } else {
            __syncthreads();
        }
        issue_kv(kt, kb);
        advance(kt, kb);
        issue_idx(xt, xb);
        advance(xt, xb);
        cp_async_commit();
        if (cb != cur_b) {
            if (cur_b >= 0) flush(cur_b);
            begin_request(cb);
            cur_b = cb;
        }
        compute_tile(i % NS, tile_k0(ct, cb));
        advance(ct, cb);
    }
    if (cur_b >= 0 && !(TMA && *abort_flag)) flush(cur_b);
    cp_async_wait<0>();
    if (TMA && tid == 0) {
        // every page load issued lands before the CTA leaves (its shared memory
        // is the destination); without an abort they all have
        for (int tile = i; tile < n_issued; ++tile)
            wait_bounded(STAGE_BAR(tile % NS), (tile / NS) & 1, abort_flag, false, TEARDOWN_LIMIT_NS);
        if (*abort_flag) {
            pdl_wait_primary();  // the step's first kernel has cleared the status word
            atomicOr(p.status, STATUS_ATTN_WAIT);
        }
    }
    pdl_launch_dependents();
}

}  // namespace gad
