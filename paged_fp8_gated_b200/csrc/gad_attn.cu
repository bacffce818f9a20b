// gad_attn.cu - C ABI of libgad_attn.so: argument checks, workspace layout and
// the three launches (prep -> decode -> combine, chained with programmatic
// dependent launch so each kernel's launch latency hides behind the previous
// kernel's tail).
//
// Decode kernel choice (measured on B200, decode-32 full attention, KV 463 MB):
// cp.async gathers from every warp of two CTAs per SM into 128-key stages run
// at 76.6% (page size 1) / 78.8% (page size 64) of the measured HBM copy rate;
// a warp-specialised variant with one producer warp issuing 2D TMA page loads
// reached 64%, and producer-warp cp.async gathers about 55%.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "gad_attn.h"
#include "gad_error.h"
#include "gad_combine.cuh"
#include "gad_kernels.cuh"
#include "gad_oproj.cuh"
#include "gad_prefill_tc.cuh"
#include "gad_prep.cuh"
#include "gad_verify_tc.cuh"

namespace {
thread_local std::string g_last_error;
}  // namespace

int gad_fail(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

namespace {

#define fail gad_fail

constexpr int kMaxCtasPerSm = 2;
constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// decode_kernel configuration for single-token steps: 128-key stages, 3 of
// them, two CTAs per SM (so 128 KB of loads in flight per SM); each of the 4
// key groups writes its own partial (no merge buffer, so the stages fit).
// Verify blocks (L > 1) run verify_tc_kernel (tcgen05), one CTA per SM.
constexpr int kV1SingleKG = 4, kV1SingleNS = 3, kV1SingleTK = 128;

// Workspace layout.  The first 256 bytes hold the step's status word (offset
// 0, read back by gad_attn_step_status); the rest is the step's scratch.
struct WsLayout {
    size_t status_off, q_off, po_off, pml_off, meta_off, total;
};

// How a step's tokens and heads become tile-list items.  Blocks longer than
// GAD_MAX_L (prefill) run prefill_tc_kernel on items (request, 32-token
// chunk, KV head) whose partial rows hold 32 tokens x 8 heads; other steps
// run decode_kernel or verify_tc_kernel on items (request, head group) with
// partial rows of up to 8 tokens x 16 heads.
struct StepShape {
    bool prefill;
    int chunk, nchunk, nsub, hp, lt;
    long long NB;
};
StepShape shape_of(int B, int L, int ngrp) {
    StepShape sh{};
    sh.prefill = L > GAD_MAX_L;
    sh.chunk = sh.prefill ? gad::PF_CHUNK : gad::CHUNK;
    sh.nchunk = (L + sh.chunk - 1) / sh.chunk;
    sh.nsub = sh.prefill ? GAD_HKV : ngrp;
    sh.hp = sh.prefill ? gad::GRP : gad::HQ;
    sh.lt = sh.prefill ? gad::PF_CHUNK : (L == 1 ? 1 : gad::CHUNK);
    sh.NB = static_cast<long long>(B) * sh.nchunk * sh.nsub;
    return sh;
}

// Partial slots: (CTAs + NB) * partials per (CTA, list item), each holding lt
// tokens x hp heads x (64 values + max + sum).
WsLayout ws_layout(int B, int L, int ngrp, int sms) {
    WsLayout w{};
    const StepShape sh = shape_of(B, L, ngrp);
    const size_t NB = static_cast<size_t>(sh.NB);
    const size_t units =
        (static_cast<size_t>(sms) * kMaxCtasPerSm + NB) * (L == 1 ? kV1SingleKG : 1);
    const size_t T = static_cast<size_t>(B) * L;
    const size_t parts = units * sh.lt * sh.hp;
    size_t off = 0;
    w.status_off = off;
    off = align_up(off + sizeof(int));
    w.q_off = off;
    off = align_up(off + T * ngrp * GAD_HQ * GAD_HEAD_DIM * 2);
    w.po_off = off;
    off = align_up(off + parts * GAD_HEAD_DIM * 4);
    w.pml_off = off;
    off = align_up(off + parts * 2 * 4);
    w.meta_off = off;
    off = align_up(off + (gad::META_INTS + NB) * 4);
    w.total = off;
    return w;
}

int current_device_sms(int* sms, int* major) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    e = cudaDeviceGetAttribute(major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    return GAD_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A driver entry point by name (nullptr if the driver does not export it).
void* driver_fn(const char* name) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return f;
}

// Unique id of the calling thread's current CUDA context, 0 if there is none
// yet or the driver cannot say.  Per-device set-up done once (function
// attributes, device-symbol addresses) is remembered together with this id,
// so a new context on the device (after cudaDeviceReset, say) repeats it.
unsigned long long current_ctx_id() {
    static std::atomic<PFN_cuCtxGetCurrent_v4000> get_cur{nullptr};
    static std::atomic<PFN_cuCtxGetId_v12000> get_id{nullptr};
    PFN_cuCtxGetCurrent_v4000 gc = get_cur.load(std::memory_order_acquire);
    PFN_cuCtxGetId_v12000 gi = get_id.load(std::memory_order_acquire);
    if (gc == nullptr || gi == nullptr) {
        gc = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(driver_fn("cuCtxGetCurrent"));
        gi = reinterpret_cast<PFN_cuCtxGetId_v12000>(driver_fn("cuCtxGetId"));
        if (gc == nullptr || gi == nullptr) return 0;
        get_cur.store(gc, std::memory_order_release);
        get_id.store(gi, std::memory_order_release);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (gc(&ctx) != CUDA_SUCCESS || ctx == nullptr || gi(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// One-time set-up per (device, context): `done[dev]` holds the id of the
// context in which it last ran.
struct OncePerContext {
    std::atomic<unsigned long long> done[kMaxDevices];
    bool is_done(int dev, unsigned long long ctx) const {
        return ctx != 0 && done[dev].load(std::memory_order_acquire) == ctx;
    }
    void mark(int dev) { done[dev].store(current_ctx_id(), std::memory_order_release); }
};

// The current device index, checked against the per-device tables.
int current_device(int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (*dev < 0 || *dev >= kMaxDevices) return fail(GAD_ERR_DEVICE, "device index %d", *dev);
    return GAD_OK;
}

cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    std::memset(&a, 0, sizeof(a));
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

// cuTensorMapEncodeTiled, looked up once through the runtime.
int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> encode{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode.load(std::memory_order_acquire);
    if (fn == nullptr) {
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(driver_fn("cuTensorMapEncodeTiled"));
        if (fn == nullptr) return fail(GAD_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        encode.store(fn, std::memory_order_release);
    }
    *out = fn;
    return GAD_OK;
}

// A cache (K or V) as a 2D byte tensor of num_rows rows of row_bytes, read in
// tiles of one 64-row page x 128 bytes (one head group) with the 128-byte
// swizzle.
int encode_cache_pages(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t num_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    const int st = tensor_map_encoder(&fn);
    if (st != GAD_OK) return st;
    const cuuint64_t dims[2] = {row_bytes, num_rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {128, 64};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GAD_ERR_CUDA, "cuTensorMapEncodeTiled (cache pages) failed (%d)", static_cast<int>(r));
    return GAD_OK;
}

template <int LT, int PS, int KG, int NS, int MINB, int TK, bool MERGE, bool MULTI>
int launch_decode(const gad::StepParams& prm, int sms, int tiles_upper, cudaStream_t stream,
                  bool pdl) {
    using C = gad::DecodeCfg<LT, KG, NS, TK, MERGE>;
    auto kern = gad::decode_kernel<LT, PS, KG, NS, MINB, TK, MERGE, MULTI>;
    const size_t smem = C::smem_bytes(prm.NB);
    // Raise the kernel's dynamic shared-memory limit once per device, to the
    // largest size any item count needs, so no attribute call happens during capture.
    static OncePerContext attr_done;
    int dev = 0;
    {
        const int ds = current_device(&dev);
        if (ds != GAD_OK) return ds;
    }
    cudaError_t e;
    if (!attr_done.is_done(dev, current_ctx_id())) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(C::smem_bytes(GAD_MAX_B)));
        if (e != cudaSuccess)
            return fail(GAD_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_done.mark(dev);
    }
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, gad::DEC_THREADS, smem);
    if (e != cudaSuccess || occ < 1)
        return fail(GAD_ERR_CUDA, "decode kernel does not fit on an SM (smem %zu B): %s", smem,
                    cudaGetErrorString(e));
    occ = occ > kMaxCtasPerSm ? kMaxCtasPerSm : occ;
    long long grid = static_cast<long long>(sms) * occ;
    if (grid > tiles_upper) grid = tiles_upper;
    if (grid < 1) grid = 1;
    CUtensorMap kmap, vmap;  // page size 64: the caches' pages, read by TMA tile loads
    std::memset(&kmap, 0, sizeof(kmap));
    std::memset(&vmap, 0, sizeof(vmap));
    if (PS == 64) {
        const uint64_t row_bytes = static_cast<uint64_t>(GAD_ROW_BYTES) * prm.ngrp;
        int st = encode_cache_pages(&kmap, prm.k_cache, row_bytes, static_cast<uint64_t>(prm.num_rows));
        if (st != GAD_OK) return st;
        st = encode_cache_pages(&vmap, prm.v_cache, row_bytes, static_cast<uint64_t>(prm.num_rows));
        if (st != GAD_OK) return st;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(gad::DEC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr = pdl_attr();
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return GAD_OK;
}

// Verify blocks (L > 1) on the tcgen05 kernel: one CTA per SM; as many raw
// stages as the shared memory leaves room for next to the per-request tables.
// Page size 64: each tile's K and V pages are read by TMA tile loads.
template <int PS, int NS, bool MULTI>
int launch_verify_tc(const gad::StepParams& prm, int sms, int tiles_upper, cudaStream_t stream,
                     bool pdl) {
    using C = gad::vtc::Cfg<NS>;
    auto kern = gad::verify_tc_kernel<PS, NS, MULTI>;
    CUtensorMap kmap, vmap;
    std::memset(&kmap, 0, sizeof(kmap));
    std::memset(&vmap, 0, sizeof(vmap));
    if (PS == 64) {
        const uint64_t row_bytes = static_cast<uint64_t>(GAD_ROW_BYTES) * prm.ngrp;
        int st = encode_cache_pages(&kmap, prm.k_cache, row_bytes, static_cast<uint64_t>(prm.num_rows));
        if (st != GAD_OK) return st;
        st = encode_cache_pages(&vmap, prm.v_cache, row_bytes, static_cast<uint64_t>(prm.num_rows));
        if (st != GAD_OK) return st;
    }
    const size_t smem = C::smem_bytes(prm.NB);
    static OncePerContext attr_done;
    int dev = 0;
    {
        const int ds = current_device(&dev);
        if (ds != GAD_OK) return ds;
    }
    cudaError_t e;
    if (!attr_done.is_done(dev, current_ctx_id())) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess)
            return fail(GAD_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e != cudaSuccess)
            return fail(GAD_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_done.mark(dev);
    }
    long long grid = sms;
    if (grid > tiles_upper) grid = tiles_upper;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(gad::vtc::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr = pdl_attr();
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, prm, kmap, vmap);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "verify launch: %s", cudaGetErrorString(e));
    return GAD_OK;
}

// Whether the deep-ring verify kernel's shared memory, with tables for NB list
// items, fits in `optin` bytes.
constexpr int kVtcDeepStages = 6, kVtcShallowStages = 3;

bool verify_deep_fits(int NB, int optin) {
    return gad::vtc::Cfg<kVtcDeepStages>::smem_bytes(NB) <= static_cast<size_t>(optin);
}

// Shape checks shared by the entry points: B, L (at most max_L), the head
// counts the kernels take (groups of 16 query heads over 2 KV heads) and the
// number of tile-list items.  Sets *ngrp, or returns an error status.
int check_shape(int B, int L, int max_L, int hq, int hkv, int* ngrp) {
    if (B < 1 || B > GAD_MAX_B) return fail(GAD_ERR_SHAPE, "B=%d not in [1,%d]", B, GAD_MAX_B);
    if (L < 1 || L > max_L) return fail(GAD_ERR_SHAPE, "L=%d not in [1,%d]", L, max_L);
    if (hkv < GAD_HKV || hkv % GAD_HKV != 0 || hq != hkv * (GAD_HQ / GAD_HKV))
        return fail(GAD_ERR_UNSUPPORTED,
                    "hq=%d, hkv=%d: supported head counts are hkv a positive multiple of %d and "
                    "hq = %d hkv", hq, hkv, GAD_HKV, GAD_HQ / GAD_HKV);
    *ngrp = hkv / GAD_HKV;
    if (L > GAD_MAX_L && *ngrp != 1)
        return fail(GAD_ERR_UNSUPPORTED, "blocks longer than %d tokens take %d query and %d KV heads",
                    GAD_MAX_L, GAD_HQ, GAD_HKV);
    const StepShape sh = shape_of(B, L, *ngrp);
    if (sh.NB > GAD_MAX_B)
        return fail(GAD_ERR_SHAPE,
                    "B=%d requests x %d chunks of %d tokens x %d = %lld tile-list items exceeds %d",
                    B, sh.nchunk, sh.chunk, sh.nsub, sh.NB, GAD_MAX_B);
    return GAD_OK;
}

size_t workspace_bytes(int B, int L, int max_L, int hq, int hkv) {
    int ngrp = 0;
    if (check_shape(B, L, max_L, hq, hkv, &ngrp) != GAD_OK) return 0;
    int sms = 0, major = 0;
    if (current_device_sms(&sms, &major) != GAD_OK) return 0;
    return ws_layout(B, L, ngrp, sms).total;
}

// Prefill blocks on the tcgen05 prefill kernel: one CTA per SM.
constexpr int kPtcStages = 6;
template <int PS>
int launch_prefill_tc(const gad::StepParams& prm, int sms, int tiles_upper, cudaStream_t stream,
                      bool pdl) {
    using C = gad::ptc::Cfg<kPtcStages>;
    auto kern = gad::prefill_tc_kernel<PS, kPtcStages>;
    const size_t smem = C::smem_bytes(prm.NB);
    static OncePerContext attr_done;
    int dev = 0;
    {
        const int ds = current_device(&dev);
        if (ds != GAD_OK) return ds;
    }
    cudaError_t e;
    if (!attr_done.is_done(dev, current_ctx_id())) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(C::smem_bytes(GAD_MAX_B)));
        if (e != cudaSuccess)
            return fail(GAD_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_done.mark(dev);
    }
    long long grid = sms;
    if (grid > tiles_upper) grid = tiles_upper;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(gad::ptc::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr = pdl_attr();
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, prm);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
    return GAD_OK;
}

// Single-token steps and verify blocks, by page size (and stage count).
template <bool MULTI>
int launch_single(const gad::StepParams& prm, int page_size, int sms, int tiles_upper,
                  cudaStream_t s, bool pdl) {
    return page_size == 1
               ? launch_decode<1, 1, kV1SingleKG, kV1SingleNS, 2, kV1SingleTK, false, MULTI>(
                     prm, sms, tiles_upper, s, pdl)
               : launch_decode<1, 64, kV1SingleKG, kV1SingleNS, 2, kV1SingleTK, false, MULTI>(
                     prm, sms, tiles_upper, s, pdl);
}

template <bool MULTI>
int launch_block(const gad::StepParams& prm, int page_size, bool deep, int sms, int tiles_upper,
                 cudaStream_t s, bool pdl) {
    if (page_size == 1)
        return deep ? launch_verify_tc<1, kVtcDeepStages, MULTI>(prm, sms, tiles_upper, s, pdl)
                    : launch_verify_tc<1, kVtcShallowStages, MULTI>(prm, sms, tiles_upper, s, pdl);
    return deep ? launch_verify_tc<64, kVtcDeepStages, MULTI>(prm, sms, tiles_upper, s, pdl)
                : launch_verify_tc<64, kVtcShallowStages, MULTI>(prm, sms, tiles_upper, s, pdl);
}

// ---------------------------------------------------------------------------
// Output projection a = out @ o^T (oproj_kernel)
// ---------------------------------------------------------------------------
// Error word of the projection kernel (a bounded wait timed out); the
// standalone entry point has no workspace to hold it.
// Status word of the standalone projection (gad_oproj), which has no
// workspace to hold it; read and cleared by gad_oproj_status.
__device__ int g_oproj_err;

int encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                   uint32_t box_outer) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    const int st = tensor_map_encoder(&fn);
    if (st != GAD_OK) return st;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GAD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return GAD_OK;
}

int check_oproj(const void* out, const void* w, const void* a, int T, int K, int N) {
    if (!out || !w || !a) return fail(GAD_ERR_NULL, "out, o_weight and a must be non-NULL");
    if (T < 1 || T > GAD_MAX_OPROJ_T) return fail(GAD_ERR_SHAPE, "T=%d not in [1,%d]", T, GAD_MAX_OPROJ_T);
    if (K < gad::opj::BK || K % gad::opj::BK != 0 || K > 65536)
        return fail(GAD_ERR_SHAPE, "K=%d must be a positive multiple of %d (at most 65536)", K, gad::opj::BK);
    if (N < gad::opj::BM || N % gad::opj::BM != 0 || N > 65536 * gad::opj::BM)
        return fail(GAD_ERR_SHAPE, "N=%d must be a positive multiple of %d", N, gad::opj::BM);
    if (!aligned(out, 16) || !aligned(w, 16) || !aligned(a, 16))
        return fail(GAD_ERR_ALIGN, "out, o_weight and a must be 16-byte aligned");
    return GAD_OK;
}

// Device address of the standalone projection's status word on the current
// device (looked up once per context).
int oproj_status_word(int** out) {
    static OncePerContext looked_up;
    static std::atomic<void*> addr[kMaxDevices];
    int dev = 0;
    const int ds = current_device(&dev);
    if (ds != GAD_OK) return ds;
    if (!looked_up.is_done(dev, current_ctx_id())) {
        void* ea = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ea, g_oproj_err);
        if (e != cudaSuccess || ea == nullptr)
            return fail(GAD_ERR_CUDA, "cudaGetSymbolAddress(status word): %s", cudaGetErrorString(e));
        addr[dev].store(ea, std::memory_order_release);
        looked_up.mark(dev);
    }
    *out = static_cast<int*>(addr[dev].load(std::memory_order_acquire));
    return GAD_OK;
}

// err: the status word the kernel reports a timed-out wait into (the step's
// workspace word when chained to a step, else the standalone word).
int launch_oproj(const void* out, const void* w, void* a, int T, int K, int N, cudaStream_t s, bool pdl,
                 int* err) {
    const int tt = T >= gad::opj::TT_MAX ? gad::opj::TT_MAX : (T + 15) / 16 * 16;
    const int nstg = gad::opj::stages(tt, K / gad::opj::BK);
    if (nstg < 1) return fail(GAD_ERR_SHAPE, "projection ring: %d stages", nstg);  // never launched empty
    const size_t smem = gad::opj::smem_bytes(tt, nstg);
    static OncePerContext attr_done;
    int dev = 0;
    {
        const int ds = current_device(&dev);
        if (ds != GAD_OK) return ds;
    }
    cudaError_t e;
    if (!attr_done.is_done(dev, current_ctx_id())) {
        e = cudaFuncSetAttribute(gad::oproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(1024 + gad::opj::SMEM_BUDGET + gad::opj::ctrl_bytes()));
        if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_done.mark(dev);
    }
    if (err == nullptr) {
        const int es = oproj_status_word(&err);
        if (es != GAD_OK) return es;
    }
    CUtensorMap wmap, xmap;
    int st = encode_bf16_2d(&wmap, w, static_cast<uint64_t>(K), static_cast<uint64_t>(N), gad::opj::BK,
                            gad::opj::BM);
    if (st != GAD_OK) return st;
    st = encode_bf16_2d(&xmap, out, static_cast<uint64_t>(K), static_cast<uint64_t>(T), gad::opj::BK,
                        static_cast<uint32_t>(tt));
    if (st != GAD_OK) return st;
    gad::OprojParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.a = static_cast<__nv_bfloat16*>(a);
    prm.T = T;
    prm.K = K;
    prm.N = N;
    prm.tt = tt;
    prm.nstg = nstg;
    prm.err = err;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(N / gad::opj::BM), static_cast<unsigned>((T + tt - 1) / tt));
    cfg.blockDim = dim3(gad::opj::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr = pdl_attr();
    cfg.attrs = &attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, gad::oproj_kernel, wmap, xmap, prm);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "projection launch: %s", cudaGetErrorString(e));
    return GAD_OK;
}

}  // namespace

extern "C" {

const char* gad_last_error(void) { return g_last_error.c_str(); }

const char* gad_status_string(int status) {
    switch (status) {
        case GAD_OK: return "GAD_OK";
        case GAD_ERR_NULL: return "GAD_ERR_NULL";
        case GAD_ERR_SHAPE: return "GAD_ERR_SHAPE";
        case GAD_ERR_ALIGN: return "GAD_ERR_ALIGN";
        case GAD_ERR_UNSUPPORTED: return "GAD_ERR_UNSUPPORTED";
        case GAD_ERR_WORKSPACE: return "GAD_ERR_WORKSPACE";
        case GAD_ERR_CUDA: return "GAD_ERR_CUDA";
        case GAD_ERR_DEVICE: return "GAD_ERR_DEVICE";
        case GAD_ERR_DTYPE: return "GAD_ERR_DTYPE";
        case GAD_ERR_STRIDE: return "GAD_ERR_STRIDE";
        default: return "unknown gad_status";
    }
}

size_t gad_attn_workspace_bytes_heads(int B, int L, int hq, int hkv) {
    return workspace_bytes(B, L, GAD_MAX_L, hq, hkv);
}

size_t gad_attn_prefill_workspace_bytes(int B, int L) {
    return workspace_bytes(B, L, GAD_MAX_PREFILL_L, GAD_HQ, GAD_HKV);
}

size_t gad_attn_workspace_bytes(int B, int L) {
    return gad_attn_workspace_bytes_heads(B, L, GAD_HQ, GAD_HKV);
}

static int run_step(const void* qkv, const int64_t* positions, const int32_t* page_table,
                    const int64_t* cache_loc, uint8_t* k_cache, uint8_t* v_cache,
                    const float* k_scale, const float* v_scale, int B, int L, int max_L, int hq,
                    int hkv, int max_pages, int64_t num_rows, int page_size, int window,
                    int use_rope, void* out, void* workspace, size_t workspace_bytes,
                    void* stream, void* const* events) {
    if (!qkv || !positions || !page_table || !cache_loc || !k_cache || !v_cache || !k_scale ||
        !v_scale || !out)
        return fail(GAD_ERR_NULL, "a required pointer is NULL");
    if (!workspace) return fail(GAD_ERR_WORKSPACE, "workspace is NULL");
    int ngrp = 0;
    {
        const int hs = check_shape(B, L, max_L, hq, hkv, &ngrp);
        if (hs != GAD_OK) return hs;
    }
    const StepShape sh = shape_of(B, L, ngrp);
    if (max_pages < 1) return fail(GAD_ERR_SHAPE, "max_pages=%d < 1", max_pages);
    if (page_size != 1 && page_size != 64)
        return fail(GAD_ERR_UNSUPPORTED, "page_size=%d (supported: 1, 64)", page_size);
    if (num_rows < 1 || num_rows % page_size != 0)
        return fail(GAD_ERR_SHAPE, "num_rows=%lld must be a positive multiple of page_size",
                    static_cast<long long>(num_rows));
    if (static_cast<long long>(max_pages) * page_size > INT32_MAX)
        return fail(GAD_ERR_SHAPE, "max_pages * page_size exceeds 2^31");
    if (num_rows > INT32_MAX)
        return fail(GAD_ERR_SHAPE, "num_rows=%lld exceeds 2^31", static_cast<long long>(num_rows));
    if (window < 0) return fail(GAD_ERR_UNSUPPORTED, "window=%d < 0", window);
    if (!aligned(qkv, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(GAD_ERR_ALIGN, "qkv, out, k_cache and v_cache must be 16-byte aligned");
    if (!aligned(positions, 8) || !aligned(cache_loc, 8) || !aligned(page_table, 4) ||
        !aligned(k_scale, 4) || !aligned(v_scale, 4))
        return fail(GAD_ERR_ALIGN, "positions/cache_loc need 8-byte, page_table/scales 4-byte alignment");
    if (!aligned(workspace, kAlign)) return fail(GAD_ERR_ALIGN, "workspace must be 256-byte aligned");

    int sms = 0, major = 0;
    int st = current_device_sms(&sms, &major);
    if (st != GAD_OK) return st;
    if (major != 10) return fail(GAD_ERR_DEVICE, "compute capability %d.x; this build targets sm_100a", major);
    const WsLayout w = ws_layout(B, L, ngrp, sms);
    if (workspace_bytes < w.total)
        return fail(GAD_ERR_WORKSPACE, "workspace %zu B < required %zu B", workspace_bytes, w.total);

    gad::StepParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.qkv = static_cast<const __nv_bfloat16*>(qkv);
    prm.positions = positions;
    prm.page_table = page_table;
    prm.cache_loc = cache_loc;
    prm.k_cache = k_cache;
    prm.v_cache = v_cache;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.B = B;
    prm.L = L;
    prm.ngrp = ngrp;
    prm.chunk = sh.chunk;
    prm.nchunk = sh.nchunk;
    prm.nsub = sh.nsub;
    prm.hp = sh.hp;
    prm.NB = static_cast<int>(sh.NB);
    prm.max_pages = max_pages;
    prm.window = window;
    prm.use_rope = use_rope ? 1 : 0;
    {
        // RoPE frequencies theta^(-2i/64), theta = 10000, once per process
        static const struct Freqs {
            double v[gad::HD / 2];
            Freqs() {
                for (int i = 0; i < gad::HD / 2; ++i) v[i] = std::pow(10000.0, -2.0 * i / 64.0);
            }
        } freqs;
        std::memcpy(prm.inv_freq, freqs.v, sizeof(prm.inv_freq));
    }
    prm.num_rows = num_rows;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    prm.q_ws = reinterpret_cast<__half*>(ws + w.q_off);
    prm.part_o = reinterpret_cast<float*>(ws + w.po_off);
    prm.part_ml = reinterpret_cast<float*>(ws + w.pml_off);
    prm.meta = reinterpret_cast<int*>(ws + w.meta_off);
    prm.status = reinterpret_cast<int*>(ws + w.status_off);

    prm.lt = sh.lt;
    prm.tl = L == 1 ? kV1SingleKG : 1;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = B * L;

    // upper bound of tiles in the step (only caps the grid; the split itself is on device)
    long long per_req;
    if (window > 0) per_req = (static_cast<long long>(window) + L - 1 + gad::TILE - 1) / gad::TILE + 1;
    else per_req = (static_cast<long long>(max_pages) * page_size + gad::TILE - 1) / gad::TILE + 1;
    long long tiles_upper_ll = per_req * prm.NB;
    const int tiles_upper = tiles_upper_ll > INT32_MAX ? INT32_MAX : static_cast<int>(tiles_upper_ll);

    const bool timed = events != nullptr;
    cudaError_t e;
    if (timed) {
        e = cudaEventRecord(static_cast<cudaEvent_t>(events[0]), s);
        if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(e));
    }
    gad::prep_kernel<<<T * ngrp, gad::PREP_THREADS, 0, s>>>(prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "prep launch: %s", cudaGetErrorString(e));
    if (timed) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), s);

    if (sh.prefill) {
        st = page_size == 1 ? launch_prefill_tc<1>(prm, sms, tiles_upper, s, !timed)
                            : launch_prefill_tc<64>(prm, sms, tiles_upper, s, !timed);
    } else if (L == 1) {
        st = prm.NB != B ? launch_single<true>(prm, page_size, sms, tiles_upper, s, !timed)
                         : launch_single<false>(prm, page_size, sms, tiles_upper, s, !timed);
    } else {
        int optin = 0, dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return fail(GAD_ERR_CUDA, "shared-memory opt-in query failed");
        const bool deep = verify_deep_fits(prm.NB, optin);
        st = prm.NB != B ? launch_block<true>(prm, page_size, deep, sms, tiles_upper, s, !timed)
                         : launch_block<false>(prm, page_size, deep, sms, tiles_upper, s, !timed);
    }
    if (st != GAD_OK) return st;
    if (timed) cudaEventRecord(static_cast<cudaEvent_t>(events[2]), s);

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(T) * gad::HQ * ngrp);
    cfg.stream = s;
    cudaLaunchAttribute attr = pdl_attr();
    cfg.attrs = &attr;
    cfg.numAttrs = timed ? 0 : 1;
    if (sh.prefill) {  // one warp per (token, head)
        constexpr int per_block = gad::COMBW_THREADS / 32;
        cfg.gridDim = dim3(static_cast<unsigned>((static_cast<long long>(T) * gad::HQ * ngrp +
                                                  per_block - 1) / per_block));
        cfg.blockDim = dim3(gad::COMBW_THREADS);
        e = cudaLaunchKernelEx(&cfg, gad::combine_warp_kernel, prm);
    } else if (T * ngrp <= 16) {
        cfg.blockDim = dim3(1024);
        e = T * gad::HQ * ngrp <= sms ? cudaLaunchKernelEx(&cfg, gad::combine_kernel<1024, 1>, prm)
                                      : cudaLaunchKernelEx(&cfg, gad::combine_kernel<1024, 2>, prm);
    } else if (L > 1) {  // verify blocks: one warp per (token, head), four slots at a time
        constexpr int per_block = gad::COMBW4_THREADS / 32;
        cfg.gridDim = dim3(static_cast<unsigned>((static_cast<long long>(T) * gad::HQ * ngrp +
                                                  per_block - 1) / per_block));
        cfg.blockDim = dim3(gad::COMBW4_THREADS);
        e = cudaLaunchKernelEx(&cfg, gad::combine_warp4_kernel, prm);
    } else {
        cfg.blockDim = dim3(256);
        e = cudaLaunchKernelEx(&cfg, gad::combine_kernel<256, 8>, prm);
    }
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
    if (timed) {
        e = cudaEventRecord(static_cast<cudaEvent_t>(events[3]), s);
        if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(e));
    }
    return GAD_OK;
}

int gad_attn_decode(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                    const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                    uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                    int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                    void* out, void* workspace, size_t workspace_bytes, void* stream) {
    (void)seq_lens;
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size, window,
                    use_rope, out,
                    workspace, workspace_bytes, stream, nullptr);
}

int gad_attn_decode_heads(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                          int L, int hq, int hkv, int max_pages, int64_t num_rows, int page_size,
                          int window, int use_rope, void* out, void* workspace,
                          size_t workspace_bytes, void* stream) {
    (void)seq_lens;
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_L, hq, hkv, max_pages, num_rows, page_size, window, use_rope, out,
                    workspace,
                    workspace_bytes, stream, nullptr);
}

int gad_attn_decode_timed(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                          int L, int max_pages, int64_t num_rows, int page_size, int window,
                          int use_rope, void* out, void* workspace, size_t workspace_bytes,
                          void* stream, void* const* events) {
    (void)seq_lens;
    if (!events || !events[0] || !events[1] || !events[2] || !events[3])
        return fail(GAD_ERR_NULL, "events must hold four cudaEvent_t");
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size, window,
                    use_rope, out,
                    workspace, workspace_bytes, stream, events);
}

int gad_attn_decode_heads_timed(const void* qkv, const int64_t* positions,
                                const int32_t* seq_lens, const int32_t* page_table,
                                const int64_t* cache_loc, uint8_t* k_cache, uint8_t* v_cache,
                                const float* k_scale, const float* v_scale, int B, int L, int hq,
                                int hkv, int max_pages, int64_t num_rows, int page_size,
                                int window, int use_rope, void* out, void* workspace,
                                size_t workspace_bytes, void* stream, void* const* events) {
    (void)seq_lens;
    if (!events || !events[0] || !events[1] || !events[2] || !events[3])
        return fail(GAD_ERR_NULL, "events must hold four cudaEvent_t");
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_L, hq, hkv, max_pages, num_rows, page_size, window, use_rope, out,
                    workspace,
                    workspace_bytes, stream, events);
}

int gad_oproj(const void* out, const void* o_weight, void* a, int T, int K, int N, void* stream) {
    const int st = check_oproj(out, o_weight, a, T, K, N);
    if (st != GAD_OK) return st;
    return launch_oproj(out, o_weight, a, T, K, N, static_cast<cudaStream_t>(stream), false, nullptr);
}

int gad_attn_decode_oproj(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                          const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                          uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                          int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                          void* out, void* workspace, size_t workspace_bytes, const void* o_weight,
                          int hidden, void* a, void* stream) {
    (void)seq_lens;
    if (L < 1 || L > GAD_MAX_PREFILL_L) return fail(GAD_ERR_SHAPE, "L=%d not in [1,%d]", L, GAD_MAX_PREFILL_L);
    if (B < 1 || B > GAD_MAX_B) return fail(GAD_ERR_SHAPE, "B=%d not in [1,%d]", B, GAD_MAX_B);
    int st = check_oproj(out, o_weight, a, B * L, GAD_OUT_COLS, hidden);
    if (st != GAD_OK) return st;
    st = run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B, L,
                  GAD_MAX_PREFILL_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size, window, use_rope,
                  out, workspace, workspace_bytes, stream, nullptr);
    if (st != GAD_OK) return st;
    return launch_oproj(out, o_weight, a, B * L, GAD_OUT_COLS, hidden, static_cast<cudaStream_t>(stream),
                        true, static_cast<int*>(workspace));  // the step's status word (offset 0)
}

int gad_attn_prefill(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                     const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                     uint8_t* v_cache, const float* k_scale, const float* v_scale, int B, int L,
                     int max_pages, int64_t num_rows, int page_size, int window, int use_rope,
                     void* out, void* workspace, size_t workspace_bytes, void* stream) {
    (void)seq_lens;
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_PREFILL_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size,
                    window, use_rope, out, workspace, workspace_bytes, stream, nullptr);
}

int gad_attn_prefill_timed(const void* qkv, const int64_t* positions, const int32_t* seq_lens,
                           const int32_t* page_table, const int64_t* cache_loc, uint8_t* k_cache,
                           uint8_t* v_cache, const float* k_scale, const float* v_scale, int B,
                           int L, int max_pages, int64_t num_rows, int page_size, int window,
                           int use_rope, void* out, void* workspace, size_t workspace_bytes,
                           void* stream, void* const* events) {
    (void)seq_lens;
    if (!events || !events[0] || !events[1] || !events[2] || !events[3])
        return fail(GAD_ERR_NULL, "events must hold four cudaEvent_t");
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_PREFILL_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size,
                    window, use_rope, out, workspace, workspace_bytes, stream, events);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant.
//
// Some callers cannot hand the library a device workspace: code running
// inside a framework whose memory pool owns every device allocation, plugins
// that may not call cudaMalloc (which can synchronise the device and is not
// allowed while another thread captures a CUDA graph), and plain C hosts with
// no device allocator of their own.  For them the step's scratch lives in one
// fixed, file-scope device array that the library carries.  Every GPU that
// loads this library holds GAD_NOALLOC_SCRATCH_BYTES of it until the process
// exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[GAD_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current, once per context, and remembered.
static int noalloc_scratch_address(void** out) {
    static OncePerContext looked_up;
    static std::atomic<void*> addr[kMaxDevices];
    int dev = 0;
    const int ds = current_device(&dev);
    if (ds != GAD_OK) return ds;
    if (!looked_up.is_done(dev, current_ctx_id())) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(GAD_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        addr[dev].store(p, std::memory_order_release);
        looked_up.mark(dev);
    }
    *out = addr[dev].load(std::memory_order_acquire);
    return GAD_OK;
}

extern "C" int gad_attn_decode_noalloc(const void* qkv, const int64_t* positions,
                                       const int32_t* seq_lens, const int32_t* page_table,
                                       const int64_t* cache_loc, uint8_t* k_cache,
                                       uint8_t* v_cache, const float* k_scale,
                                       const float* v_scale, int B, int L, int max_pages,
                                       int64_t num_rows, int page_size, int window, int use_rope,
                                       void* out, void* stream) {
    (void)seq_lens;
    const size_t need = gad_attn_workspace_bytes(B, L);
    if (need == 0) return B < 1 || B > GAD_MAX_B || L < 1 || L > GAD_MAX_L ? GAD_ERR_SHAPE : GAD_ERR_CUDA;
    if (need > static_cast<size_t>(GAD_NOALLOC_SCRATCH_BYTES))
        return fail(GAD_ERR_WORKSPACE,
                    "B=%d, L=%d needs %zu B of scratch but the built-in scratch holds %zu B; "
                    "call gad_attn_decode with a caller workspace instead",
                    B, L, need, static_cast<size_t>(GAD_NOALLOC_SCRATCH_BYTES));
    void* scratch = nullptr;
    const int st = noalloc_scratch_address(&scratch);
    if (st != GAD_OK) return st;
    return run_step(qkv, positions, page_table, cache_loc, k_cache, v_cache, k_scale, v_scale, B,
                    L, GAD_MAX_L, GAD_HQ, GAD_HKV, max_pages, num_rows, page_size, window,
                    use_rope, out,
                    scratch, static_cast<size_t>(GAD_NOALLOC_SCRATCH_BYTES), stream, nullptr);
}

// ---------------------------------------------------------------------------
// Status words: a kernel whose bounded wait gave up (a stalled pipeline) sets
// a bit in its step's status word instead of hanging; these calls bring the
// word back to the host.
// ---------------------------------------------------------------------------
extern "C" int gad_attn_step_status(const void* workspace, int* status, void* stream) {
    if (!status) return fail(GAD_ERR_NULL, "status must point to a host int");
    const void* word = workspace;
    if (word == nullptr) {
        void* scratch = nullptr;
        const int st = noalloc_scratch_address(&scratch);
        if (st != GAD_OK) return st;
        word = scratch;
    } else if (!aligned(workspace, kAlign)) {
        return fail(GAD_ERR_ALIGN, "workspace must be 256-byte aligned");
    }
    cudaError_t e = cudaMemcpyAsync(status, word, sizeof(int), cudaMemcpyDeviceToHost,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "cudaMemcpyAsync(status): %s", cudaGetErrorString(e));
    return GAD_OK;
}

extern "C" int gad_oproj_status(int* status, void* stream) {
    if (!status) return fail(GAD_ERR_NULL, "status must point to a host int");
    int* word = nullptr;
    const int st = oproj_status_word(&word);
    if (st != GAD_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(status, word, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(int), s);
    if (e != cudaSuccess) return fail(GAD_ERR_CUDA, "projection status: %s", cudaGetErrorString(e));
    return GAD_OK;
}
