// gad_desc.cu - the tensor-descriptor form of the step (gad_attn_decode_t):
// every argument arrives as a gad_tensor (data pointer, element type, shape,
// strides), is checked against the layouts the step takes, and the call is
// forwarded to the plain-pointer entry points in gad_attn.cu.  Also the
// per-device workspace registry the descriptor form draws its scratch from.
//
// The shapes are those of the task page "Gated attention decode
// (muse_attention_decode)", section "Shapes" (16 query heads, 2 KV heads,
// head dim 64 per GPU; "heads dp" multiples of them), with the inputs the
// serving stack hands the attention kernel listed there: the fused qkv rows,
// positions, cache rows, lengths, page table, caches and their scales.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "gad_attn.h"
#include "gad_error.h"

namespace {

constexpr int kMaxDevices = 64;

// Records the message gad_last_error() returns and passes the status through.
#define desc_fail gad_fail

struct Registered {
    std::atomic<void*> ptr{nullptr};
    std::atomic<size_t> bytes{0};
};
Registered g_ws[kMaxDevices];

const char* dtype_name(int32_t d) {
    switch (d) {
        case GAD_DTYPE_BF16: return "bf16";
        case GAD_DTYPE_E4M3: return "e4m3";
        case GAD_DTYPE_U8: return "u8";
        case GAD_DTYPE_I32: return "i32";
        case GAD_DTYPE_I64: return "i64";
        case GAD_DTYPE_F32: return "f32";
        default: return "unknown";
    }
}

// Checks one descriptor: non-NULL data, element type, rank, the extents given
// in `shape` (-1: any positive extent, returned in `got`) and densely packed
// row-major strides.
int check(const gad_tensor* t, const char* name, int32_t dtype, int32_t alt_dtype, int ndim,
          const int64_t* shape, int64_t* got) {
    if (t == nullptr || t->data == nullptr) return desc_fail(GAD_ERR_NULL, "%s: NULL descriptor or data", name);
    if (t->dtype != dtype && t->dtype != alt_dtype)
        return desc_fail(GAD_ERR_DTYPE, "%s: element type %s (%d), expected %s", name, dtype_name(t->dtype),
                         t->dtype, dtype_name(dtype));
    if (t->ndim != ndim)
        return desc_fail(GAD_ERR_SHAPE, "%s: %d dimensions, expected %d", name, t->ndim, ndim);
    for (int i = 0; i < ndim; ++i) {
        if (t->shape[i] < 1)
            return desc_fail(GAD_ERR_SHAPE, "%s: extent %lld in dimension %d", name,
                             static_cast<long long>(t->shape[i]), i);
        if (shape[i] >= 0 && t->shape[i] != shape[i])
            return desc_fail(GAD_ERR_SHAPE, "%s: extent %lld in dimension %d, expected %lld", name,
                             static_cast<long long>(t->shape[i]), i, static_cast<long long>(shape[i]));
        got[i] = t->shape[i];
    }
    int64_t expect = 1;
    for (int i = ndim - 1; i >= 0; --i) {
        if (t->stride[i] != expect)
            return desc_fail(GAD_ERR_STRIDE, "%s: stride %lld in dimension %d, expected %lld (densely packed, "
                             "row-major)", name, static_cast<long long>(t->stride[i]), i,
                             static_cast<long long>(expect));
        expect *= t->shape[i];
    }
    return GAD_OK;
}

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return desc_fail(GAD_ERR_CUDA, "cudaGetDevice failed");
    if (*dev < 0 || *dev >= kMaxDevices) return desc_fail(GAD_ERR_DEVICE, "device index %d", *dev);
    return GAD_OK;
}

}  // namespace

extern "C" {

int gad_attn_set_workspace(void* workspace, size_t bytes) {
    int dev = 0;
    const int st = current_device(&dev);
    if (st != GAD_OK) return st;
    if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return desc_fail(GAD_ERR_ALIGN, "workspace must be 256-byte aligned");
    g_ws[dev].bytes.store(workspace ? bytes : 0, std::memory_order_release);
    g_ws[dev].ptr.store(workspace, std::memory_order_release);
    return GAD_OK;
}

size_t gad_attn_workspace_bytes_t(int B, int L, int max_pages, int page_size, int window) {
    if (max_pages < 1) {
        desc_fail(GAD_ERR_SHAPE, "max_pages=%d < 1", max_pages);
        return 0;
    }
    if (page_size != 1 && page_size != 64) {
        desc_fail(GAD_ERR_UNSUPPORTED, "page_size=%d (supported: 1, 64)", page_size);
        return 0;
    }
    if (window < 0) {
        desc_fail(GAD_ERR_UNSUPPORTED, "window=%d < 0", window);
        return 0;
    }
    return L > GAD_MAX_L ? gad_attn_prefill_workspace_bytes(B, L) : gad_attn_workspace_bytes(B, L);
}

int gad_attn_decode_t(const gad_tensor* qkv, const gad_tensor* positions, const gad_tensor* seq_lens,
                      const gad_tensor* page_table, const gad_tensor* cache_loc, const gad_tensor* k_cache,
                      const gad_tensor* v_cache, const gad_tensor* k_scale, const gad_tensor* v_scale,
                      int page_size, int window, int use_rope, const gad_tensor* out, void* stream) {
    int64_t o[4], q[4], p[4], c[4], pt[4], kc[4], vc[4], s[4];
    int st;
    // out [B, L, 64 hq] bf16 gives B, L and the query heads
    {
        const int64_t any3[3] = {-1, -1, -1};
        if ((st = check(out, "out", GAD_DTYPE_BF16, GAD_DTYPE_BF16, 3, any3, o)) != GAD_OK) return st;
    }
    if (o[0] > GAD_MAX_B || o[1] > GAD_MAX_PREFILL_L)
        return desc_fail(GAD_ERR_SHAPE, "out: B=%lld, L=%lld out of range", static_cast<long long>(o[0]),
                         static_cast<long long>(o[1]));
    if (o[2] % GAD_HEAD_DIM != 0)
        return desc_fail(GAD_ERR_SHAPE, "out: %lld columns, not a multiple of %d", static_cast<long long>(o[2]),
                         GAD_HEAD_DIM);
    const int B = static_cast<int>(o[0]), L = static_cast<int>(o[1]);
    const int hq = static_cast<int>(o[2] / GAD_HEAD_DIM);
    const int64_t T = static_cast<int64_t>(B) * L;
    // qkv [T, 64 (2 hq + 2 hkv)] bf16 gives the KV heads
    {
        const int64_t sh[2] = {T, -1};
        if ((st = check(qkv, "qkv", GAD_DTYPE_BF16, GAD_DTYPE_BF16, 2, sh, q)) != GAD_OK) return st;
    }
    const int64_t spare = q[1] - 2LL * hq * GAD_HEAD_DIM;
    if (spare <= 0 || spare % (2 * GAD_HEAD_DIM) != 0)
        return desc_fail(GAD_ERR_SHAPE, "qkv: %lld columns do not hold q and gate of %d heads plus k and v heads "
                         "of 64", static_cast<long long>(q[1]), hq);
    const int hkv = static_cast<int>(spare / (2 * GAD_HEAD_DIM));
    {
        const int64_t sh[1] = {T};
        if ((st = check(positions, "positions", GAD_DTYPE_I64, GAD_DTYPE_I64, 1, sh, p)) != GAD_OK) return st;
        if ((st = check(cache_loc, "cache_loc", GAD_DTYPE_I64, GAD_DTYPE_I64, 1, sh, c)) != GAD_OK) return st;
    }
    if (seq_lens != nullptr) {
        const int64_t sh[1] = {B};
        int64_t sl[4];
        if ((st = check(seq_lens, "seq_lens", GAD_DTYPE_I32, GAD_DTYPE_I32, 1, sh, sl)) != GAD_OK) return st;
    }
    {
        const int64_t sh[2] = {B, -1};
        if ((st = check(page_table, "page_table", GAD_DTYPE_I32, GAD_DTYPE_I32, 2, sh, pt)) != GAD_OK) return st;
    }
    if (pt[1] > INT32_MAX) return desc_fail(GAD_ERR_SHAPE, "page_table: too many pages per request");
    {
        const int64_t sh[4] = {-1, page_size, hkv, GAD_HEAD_DIM};
        if ((st = check(k_cache, "k_cache", GAD_DTYPE_E4M3, GAD_DTYPE_U8, 4, sh, kc)) != GAD_OK) return st;
        if ((st = check(v_cache, "v_cache", GAD_DTYPE_E4M3, GAD_DTYPE_U8, 4, sh, vc)) != GAD_OK) return st;
    }
    if (kc[0] != vc[0]) return desc_fail(GAD_ERR_SHAPE, "k_cache and v_cache hold different page counts");
    {
        const int64_t sh[1] = {1};
        if ((st = check(k_scale, "k_scale", GAD_DTYPE_F32, GAD_DTYPE_F32, 1, sh, s)) != GAD_OK) return st;
        if ((st = check(v_scale, "v_scale", GAD_DTYPE_F32, GAD_DTYPE_F32, 1, sh, s)) != GAD_OK) return st;
    }
    if (L > GAD_MAX_L && (hq != GAD_HQ || hkv != GAD_HKV))
        return desc_fail(GAD_ERR_UNSUPPORTED, "blocks longer than %d tokens take %d query and %d KV heads",
                         GAD_MAX_L, GAD_HQ, GAD_HKV);

    int dev = 0;
    if ((st = current_device(&dev)) != GAD_OK) return st;
    void* ws = g_ws[dev].ptr.load(std::memory_order_acquire);
    const size_t ws_bytes = g_ws[dev].bytes.load(std::memory_order_acquire);
    if (ws == nullptr)
        return desc_fail(GAD_ERR_WORKSPACE, "no workspace registered for device %d (gad_attn_set_workspace)", dev);

    const int max_pages = static_cast<int>(pt[1]);
    const int64_t num_rows = kc[0] * page_size;
    const int32_t* sl = seq_lens ? static_cast<const int32_t*>(seq_lens->data) : nullptr;
    if (L > GAD_MAX_L)
        return gad_attn_prefill(qkv->data, static_cast<const int64_t*>(positions->data), sl,
                                static_cast<const int32_t*>(page_table->data),
                                static_cast<const int64_t*>(cache_loc->data), static_cast<uint8_t*>(k_cache->data),
                                static_cast<uint8_t*>(v_cache->data), static_cast<const float*>(k_scale->data),
                                static_cast<const float*>(v_scale->data), B, L, max_pages, num_rows, page_size,
                                window, use_rope, out->data, ws, ws_bytes, stream);
    return gad_attn_decode_heads(qkv->data, static_cast<const int64_t*>(positions->data), sl,
                                 static_cast<const int32_t*>(page_table->data),
                                 static_cast<const int64_t*>(cache_loc->data),
                                 static_cast<uint8_t*>(k_cache->data), static_cast<uint8_t*>(v_cache->data),
                                 static_cast<const float*>(k_scale->data),
                                 static_cast<const float*>(v_scale->data), B, L, hq, hkv, max_pages, num_rows,
                                 page_size, window, use_rope, out->data, ws, ws_bytes, stream);
}

}  // extern "C"
