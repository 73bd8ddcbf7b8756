// attn_lib.cu -- the C ABI of libattn_b200.so (declared in include/attn.h).
//
// One translation unit: the kernels are header-only (encoder.cuh, decode.cuh,
// paged.cuh, rope.cuh) and included here, so the per-device status word is a
// single static __device__ variable. Host code validates arguments, encodes TMA
// tensor maps, and launches on the caller's stream. It makes no allocation call
// (the no-alloc decode's scratch is a static __device__ array).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "decode.cuh"
#include "encoder.cuh"
#include "encoder1q.cuh"
#include "paged.cuh"
#include "proj.cuh"
#include "rope.cuh"
#include "tmap.cuh"

namespace {

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }

// Dynamic shared memory opt-in, once per (kernel, device).
template <typename K>
int ensure_smem(K kernel, int bytes, std::atomic<uint64_t>& done_mask) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    const uint64_t bit = 1ull << (dev & 63);
    if (done_mask.load(std::memory_order_acquire) & bit) return ATTN_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return ATTN_ERR_CUDA;
    done_mask.fetch_or(bit, std::memory_order_acq_rel);
    return ATTN_OK;
}

// Head dim 64: one query tile per CTA, two CTAs per SM (encoder1q.cuh), with or without a
// key bias.
template <bool kBias>
int launch_encoder1q(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int B,
                     int H, int S, float scale, const float* key_bias, cudaStream_t stream) {
    using namespace attn::enc1q;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = encoder_1q_kernel<kBias>;
    int rc = ensure_smem(kernel, kSmemBytes, smem_done);
    if (rc) return rc;
    CUtensorMap tq, tk, tv;
    const uint64_t rows = static_cast<uint64_t>(S);
    const uint64_t heads = static_cast<uint64_t>(B) * H;
    if ((rc = attn::encode_map_3d_bf16(&tq, q, kD, rows, heads, 64, kTileM))) return rc;
    if ((rc = attn::encode_map_3d_bf16(&tk, k, kD, rows, heads, 64, kTileN))) return rc;
    if ((rc = attn::encode_map_3d_bf16(&tv, v, kD, rows, heads, 64, kTileN))) return rc;
    dim3 grid((S + kTileM - 1) / kTileM, static_cast<unsigned>(heads));
    return attn::launch_pdl(kernel, grid, dim3(kThreads), kSmemBytes, stream, tq, tk, tv, out,
                            key_bias, H, S, scale * kLog2e);
}

template <int D, bool kBias>
int launch_encoder(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int B,
                   int H, int S, float scale, const float* key_bias, cudaStream_t stream) {
    using namespace attn::enc;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = encoder_fwd_kernel<D, kBias>;
    int rc = ensure_smem(kernel, Cfg<D>::kSmemBytes, smem_done);
    if (rc) return rc;
    CUtensorMap tq, tk, tv;
    const uint64_t rows = static_cast<uint64_t>(S);
    const uint64_t heads = static_cast<uint64_t>(B) * H;
    if ((rc = attn::encode_map_3d_bf16(&tq, q, D, rows, heads, 64, kTileM))) return rc;
    if ((rc = attn::encode_map_3d_bf16(&tk, k, D, rows, heads, 64, kTileN))) return rc;
    if ((rc = attn::encode_map_3d_bf16(&tv, v, D, rows, heads, 64, kTileN))) return rc;
    dim3 grid((S + kRowsPerCta - 1) / kRowsPerCta, static_cast<unsigned>(heads));
    const float scale_log2 = scale * kLog2e;
    return attn::launch_pdl(kernel, grid, dim3(kThreads), Cfg<D>::kSmemBytes, stream, tq, tk, tv, out,
                            key_bias, H, S, scale_log2);
}

// Scratch for attn_gqa_decode_noalloc: reserved statically on every device that
// loads this library, so that entry point never allocates. Host code must not
// use the symbol as an address; it looks up the device address once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};   // context the cached address belongs to

// The current driver context (the runtime's primary context of the current device once
// any runtime call has run on it), through the driver entry point the runtime exposes.
CUcontext current_context() {
    using GetCurrent = CUresult (*)(CUcontext*);
    static GetCurrent fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCurrent>(p);
    });
    CUcontext ctx = nullptr;
    if (fn) fn(&ctx);
    return ctx;
}

// Device address of g_noalloc_scratch on the current device. It is looked up once per
// device and context: after cudaDeviceReset the module is loaded again in a new primary
// context, possibly at another address, so a change of context repeats the look-up.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    // No context current on this thread yet (ctx == NULL) also repeats the look-up, which
    // makes the device's primary context current; the context is read again after it.
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = current_context();
    }
    *out = g_scratch_ptr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_version(void) { return kVersion; }

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_NULL: return "ATTN_ERR_NULL";
        case ATTN_ERR_SHAPE: return "ATTN_ERR_SHAPE";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
        case ATTN_ERR_ALIGN: return "ATTN_ERR_ALIGN";
        case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
        case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT";
        case ATTN_ERR_BLOCK_TABLE: return "ATTN_ERR_BLOCK_TABLE";
        case ATTN_ERR_SEQUENCE: return "ATTN_ERR_SEQUENCE";
        default: return "ATTN_ERR_UNKNOWN";
    }
}

int attn_check(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, attn::g_attn_device_status, sizeof(int)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(attn::g_attn_device_status, &zero, sizeof(int)) != cudaSuccess)
            return ATTN_ERR_CUDA;
    }
    return v;
}

int attn_encoder_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                     int B, int H, int S, int D, float softmax_scale, const float* key_bias,
                     void* stream) {
    if (!q || !k || !v || !out) return ATTN_ERR_NULL;
    if (B < 1 || H < 1 || S < 1 || !scale_ok(softmax_scale)) return ATTN_ERR_SHAPE;
    if (static_cast<int64_t>(B) * H > 65535) return ATTN_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_ALIGN;
    if (key_bias && (reinterpret_cast<uintptr_t>(key_bias) & 3u)) return ATTN_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (D == 64)
        return key_bias ? launch_encoder1q<true>(q, k, v, out, B, H, S, softmax_scale, key_bias, st)
                        : launch_encoder1q<false>(q, k, v, out, B, H, S, softmax_scale, nullptr, st);
    return key_bias ? launch_encoder<128, true>(q, k, v, out, B, H, S, softmax_scale, key_bias, st)
                    : launch_encoder<128, false>(q, k, v, out, B, H, S, softmax_scale, nullptr, st);
}

size_t attn_gqa_decode_workspace_size(int B, int Hq, int Hkv, int S_ctx, int D) {
    if (B < 1 || Hq < 1 || Hkv < 1 || S_ctx < 1 || D < 1 || Hq % Hkv) return 0;
    return attn::dec::workspace_bytes(B, Hq, Hkv, S_ctx, D);
}

int attn_gqa_decode(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const float* attn_mask, uint16_t* out, int B, int Hq, int Hkv,
                    int num_kv_groups, int S_ctx, int D, float softmax_scale, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !out) return ATTN_ERR_NULL;
    if (B < 1 || Hq < 1 || Hkv < 1 || S_ctx < 1 || num_kv_groups < 1) return ATTN_ERR_SHAPE;
    if (Hq != Hkv * num_kv_groups || !scale_ok(softmax_scale)) return ATTN_ERR_SHAPE;
    if (D != 128 && D != 256 && D != 512) return ATTN_ERR_UNSUPPORTED;
    if (num_kv_groups > attn::dec::kMaxGroups) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(B) * Hkv > 65535 || !attn::dec::items_fit(B, Hkv, S_ctx))
        return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_ALIGN;
    if (attn_mask && (reinterpret_cast<uintptr_t>(attn_mask) & 15u)) return ATTN_ERR_ALIGN;
    const size_t need = attn::dec::workspace_bytes(B, Hq, Hkv, S_ctx, D);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_ERR_ALIGN;
    return attn::dec::launch(q, k, v, attn_mask, out, B, Hq, Hkv, num_kv_groups, S_ctx, D,
                             softmax_scale, workspace, static_cast<cudaStream_t>(stream));
}

int attn_gqa_decode_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            const float* attn_mask, uint16_t* out, int B, int Hq, int Hkv,
                            int num_kv_groups, int S_ctx, int D, float softmax_scale,
                            void* stream) {
    if (B < 1 || Hq < 1 || Hkv < 1 || S_ctx < 1 || Hq % Hkv) return ATTN_ERR_SHAPE;
    const size_t need = attn::dec::workspace_bytes(B, Hq, Hkv, S_ctx, D);
    if (need > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    return attn_gqa_decode(q, k, v, attn_mask, out, B, Hq, Hkv, num_kv_groups, S_ctx, D,
                           softmax_scale, scratch, ATTN_NOALLOC_SCRATCH_BYTES, stream);
}

int attn_paged_history(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                       const int32_t* block_table, int n_table, int num_phys_blocks,
                       int block_size, int actual_history_len, float k_scale, float v_scale,
                       float softmax_scale, int Hq, int Hkv, int num_kv_groups, int Sq, int D,
                       uint16_t* out, void* stream) {
    if (!q || !k_cache || !v_cache || !block_table || !out) return ATTN_ERR_NULL;
    if (Hq < 1 || Hkv < 1 || num_kv_groups < 1 || Hq != Hkv * num_kv_groups || Sq < 1)
        return ATTN_ERR_SHAPE;
    if (n_table < 0 || num_phys_blocks < 1 || actual_history_len < 0) return ATTN_ERR_SHAPE;
    if (block_size < 128 || block_size > 512 || block_size % 128) return ATTN_ERR_SHAPE;
    if (static_cast<int64_t>(actual_history_len) > static_cast<int64_t>(n_table) * block_size)
        return ATTN_ERR_SHAPE;
    if (!scale_ok(softmax_scale) || !scale_ok(k_scale) || !std::isfinite(v_scale))
        return ATTN_ERR_SHAPE;
    if (D != 256) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u))
        return ATTN_ERR_ALIGN;
    return attn::paged::launch(q, k_cache, v_cache, block_table, n_table, num_phys_blocks,
                               block_size, actual_history_len, k_scale, v_scale, softmax_scale,
                               Hq, Hkv, num_kv_groups, Sq, D, out,
                               static_cast<cudaStream_t>(stream));
}

int attn_paged_prefill(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                       const int32_t* block_tables, int table_stride, int num_phys_blocks,
                       int block_size, const int32_t* q_start, const int32_t* hist_lens,
                       int num_seqs, int total_q, int max_q_len, float k_scale, float v_scale,
                       float softmax_scale, int Hq, int Hkv, int num_kv_groups, int D,
                       uint16_t* out, void* stream) {
    if (!q || !k_cache || !v_cache || !block_tables || !q_start || !hist_lens || !out)
        return ATTN_ERR_NULL;
    if (Hq < 1 || Hkv < 1 || num_kv_groups < 1 || Hq != Hkv * num_kv_groups) return ATTN_ERR_SHAPE;
    if (num_seqs < 1 || num_seqs > 65535 || total_q < 0 || max_q_len < 0 || table_stride < 1 ||
        num_phys_blocks < 1)
        return ATTN_ERR_SHAPE;
    if (block_size < 128 || block_size > 512 || block_size % 128) return ATTN_ERR_SHAPE;
    if (!scale_ok(softmax_scale) || !scale_ok(k_scale) || !std::isfinite(v_scale)) return ATTN_ERR_SHAPE;
    if (D != 256) return ATTN_ERR_UNSUPPORTED;
    if (Hq > 65535) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(q_start) & 3u) ||
        (reinterpret_cast<uintptr_t>(hist_lens) & 3u))
        return ATTN_ERR_ALIGN;
    return attn::paged::launch_prefill(q, k_cache, v_cache, block_tables, table_stride,
                                       num_phys_blocks, block_size, q_start, hist_lens, num_seqs,
                                       total_q, max_q_len, k_scale, v_scale, softmax_scale, Hq, Hkv,
                                       num_kv_groups, out, static_cast<cudaStream_t>(stream));
}

int attn_rope_qk(const uint16_t* q, const uint16_t* k, uint16_t* q_out, uint16_t* k_out,
                 const float* cos_table, const float* sin_table, int B, int H, int S, int D,
                 int interleaved, void* stream) {
    if (!q || !k || !q_out || !k_out || !cos_table || !sin_table) return ATTN_ERR_NULL;
    if (B < 1 || H < 1 || S < 1 || D < 1 || (interleaved != 0 && interleaved != 1))
        return ATTN_ERR_SHAPE;
    if (D % 16 || D > 512) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out) ||
        !aligned16(cos_table) || !aligned16(sin_table))
        return ATTN_ERR_ALIGN;
    // outputs may alias their own input exactly; any other overlap is rejected
    const size_t bytes = static_cast<size_t>(B) * H * S * D * 2;
    auto overlap = [bytes](const void* a, const void* b) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
        return x < y + bytes && y < x + bytes;
    };
    if ((q_out != q && overlap(q_out, q)) || (k_out != k && overlap(k_out, k)) ||
        overlap(q_out, k_out) || overlap(q_out, k) || overlap(k_out, q))
        return ATTN_ERR_SHAPE;
    return attn::rope::launch(q, k, q_out, k_out, cos_table, sin_table, B, H, S, D,
                              interleaved != 0, static_cast<cudaStream_t>(stream));
}

int attn_qkv_rope_proj(const uint16_t* x, const uint16_t* w_qkv, const float* b_qkv,
                       const float* cos_table, const float* sin_table, int interleaved, int B,
                       int S, int C, int H, int D, uint16_t* q, uint16_t* k, uint16_t* v,
                       void* stream) {
    if (!x || !w_qkv || !q || !k || !v) return ATTN_ERR_NULL;
    if ((cos_table == nullptr) != (sin_table == nullptr)) return ATTN_ERR_NULL;
    if (B < 1 || S < 1 || C < 1 || H < 1 || (interleaved != 0 && interleaved != 1))
        return ATTN_ERR_SHAPE;
    if ((D != 64 && D != 128) || C % 64 || (H * D) % 128 || B > 65535) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(H) * D > (1 << 20) || C > (1 << 20)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
        (b_qkv && !aligned16(b_qkv)) || (cos_table && (!aligned16(cos_table) || !aligned16(sin_table))))
        return ATTN_ERR_ALIGN;
    const int rope = cos_table ? (interleaved ? 2 : 1) : 0;
    return attn::proj::launch_qkv(x, w_qkv, b_qkv, cos_table, sin_table, rope, B, S, C, H, D, q, k,
                                  v, static_cast<cudaStream_t>(stream));
}

int attn_out_proj(const uint16_t* o, const uint16_t* w_o, const float* b_o, int B, int S, int H,
                  int D, int C_out, float* y, void* stream) {
    if (!o || !w_o || !y) return ATTN_ERR_NULL;
    if (B < 1 || S < 1 || H < 1 || C_out < 1) return ATTN_ERR_SHAPE;
    if ((D != 64 && D != 128) || C_out % 128 || B > 65535 || C_out / 128 > 65535)
        return ATTN_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(H) * D > (1 << 20)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(o) || !aligned16(w_o) || !aligned16(y) || (b_o && !aligned16(b_o)))
        return ATTN_ERR_ALIGN;
    return attn::proj::launch_out(o, w_o, b_o, B, S, H, D, C_out, y,
                                  static_cast<cudaStream_t>(stream));
}

}  // extern "C"
