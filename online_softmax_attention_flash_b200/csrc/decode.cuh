// decode.cuh -- single-token GQA flash-decode for sm_100a.
//
// What it computes ("head_dim>128 (256/512) GQA Flash-Decode NKI Kernel for
// AWS Trainium", "Input contract"): for every batch entry b and query head h,
//   out[b,h] = softmax(scale * q[b,h] K[b,g]^T + attn_mask[b]) V[b,g],
//   g = h / num_kv_groups, S_q = 1, head_dim D in {128, 256, 512}.
//
// How. Decode is bound by HBM bandwidth (every K/V byte is used by only
// num_kv_groups query heads), so the tensor cores stay idle and the design is
// about moving K/V once, at full bandwidth:
//   * split-KV (the page's "multi-program dispatch" follow-on): grid =
//     (key splits, kv heads, batch). One CTA streams `kSplitKeys` keys of one
//     (b, g) with bulk async copies (cp.async.bulk) through a shared-memory
//     ring and serves all num_kv_groups query heads of that kv head from the
//     same bytes (the pages' GQA packing, as data reuse rather than MMA rows);
//   * 32-key sub-tiles whose mask is all -inf, or that lie past S_ctx, are
//     never read (length-aware skipping);
//   * each CTA writes an unnormalised partial (o, m, l) to the workspace; a
//     second kernel combines the splits with the log-sum-exp rule.
// Scores are kept in log2 units (scale * log2 e folded into q . k) so the
// exponentials are single ex2 instructions.
#pragma once

#include "ptx.cuh"

namespace attn {
namespace dec {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSubKeys = 32;                 // keys per pipeline stage
constexpr int kSplitKeys = 256;              // keys per CTA (8 sub-tiles)
constexpr int kSubTiles = kSplitKeys / kSubKeys;
constexpr int kMaxGroups = 8;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int num_splits(int S_ctx) { return (S_ctx + kSplitKeys - 1) / kSplitKeys; }

// workspace: o partials [B, Hq, n_split, D] fp32, then m and l [B, Hq, n_split] fp32
inline size_t workspace_bytes(int B, int Hq, int S_ctx, int D) {
    const size_t rows = static_cast<size_t>(B) * Hq * num_splits(S_ctx);
    size_t o = rows * D * sizeof(float);
    size_t ml = ((rows * sizeof(float) + 255) / 256) * 256;
    return o + 2 * ml;
}

template <int D>
struct Cfg {
    static constexpr int kStages = (D <= 256) ? 3 : 2;
    static constexpr int kRowBytes = D * 2;
    static constexpr int kSubBytes = kSubKeys * kRowBytes;      // K (or V) rows of one sub-tile
    static constexpr int kStageBytes = 2 * kSubBytes;           // K then V
    static constexpr int kEPL = D / 32;                          // K elements per lane in q.k
    static constexpr int kKS = 512 / D;                          // key subsets in P.V
    static constexpr int kRingOff = 0;
    static constexpr int kScoreOff = kRingOff + kStages * kStageBytes;      // [G][32] fp32
    static constexpr int kAlphaOff = kScoreOff + kMaxGroups * kSubKeys * 4; // [G] fp32
    static constexpr int kMaskOff = kAlphaOff + kMaxGroups * 4;             // [kSplitKeys] fp32
    static constexpr int kRedOff = kMaskOff + kSplitKeys * 4;               // [KS][G][D] fp32
    static constexpr int kBarOff = kRedOff + kKS * kMaxGroups * D * 4;
    static constexpr int kMiscOff = kBarOff + kStages * 8;
    static constexpr int kSmemBytes = kMiscOff + 64;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, const float* __restrict__ mask,
                    float* __restrict__ ws_o, float* __restrict__ ws_m, float* __restrict__ ws_l,
                    int Hkv, int S_ctx, float scale_log2) {
    using C = Cfg<D>;
    extern __shared__ __align__(128) uint8_t smem[];
    float* s_score = reinterpret_cast<float*>(smem + C::kScoreOff);   // [G][32], then P
    float* s_alpha = reinterpret_cast<float*>(smem + C::kAlphaOff);
    float* s_mask = reinterpret_cast<float*>(smem + C::kMaskOff);
    float* s_red = reinterpret_cast<float*>(smem + C::kRedOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);
    int* live_list = reinterpret_cast<int*>(smem + C::kMiscOff + 4);   // kSubTiles entries
    int* n_live_sm = reinterpret_cast<int*>(smem + C::kMiscOff + 4 + 4 * kSubTiles);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hq = Hkv * G;
    const int n_split = gridDim.x;
    const int key0 = split * kSplitKeys;
    const size_t kv_base = (static_cast<size_t>(b) * Hkv + g) * S_ctx;

    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // additive mask of this split, in log2 units; -inf also past S_ctx
    {
        const int key = key0 + tid;   // kThreads == kSplitKeys
        float mv = -INFINITY;
        if (key < S_ctx) mv = mask ? mask[static_cast<size_t>(b) * S_ctx + key] * kLog2e : 0.f;
        s_mask[tid] = mv;
        const bool any = __any_sync(0xffffffffu, mv != -INFINITY);  // warp w covers sub-tile w
        if (lane == 0) live_list[warp] = any ? 1 : 0;
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0;
        for (int i = 0; i < kSubTiles; ++i)
            if (live_list[i]) live_list[n++] = i;
        *n_live_sm = n;
    }
    __syncthreads();
    const int n_live = *n_live_sm;

    auto issue = [&](int li) {   // li-th live sub-tile -> stage li % kStages
        const int st = li % C::kStages;
        const int sub = live_list[li];
        const int kk0 = key0 + sub * kSubKeys;
        const int rows = min(kSubKeys, S_ctx - kk0);
        const uint32_t bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
        uint8_t* dst = smem + C::kRingOff + st * C::kStageBytes;
        mbar_arrive_expect_tx(&full[st], 2 * bytes);
        bulk_load(dst, k + (kv_base + kk0) * D, bytes, &full[st]);
        bulk_load(dst + C::kSubBytes, v + (kv_base + kk0) * D, bytes, &full[st]);
    };
    if (tid == 0)
        for (int li = 0; li < n_live && li < C::kStages; ++li) issue(li);

    // q of the G heads of this kv head: lane's slice [lane*EPL, lane*EPL + EPL), fp32
    float qr[G][C::kEPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint16_t* qh = q + (static_cast<size_t>(b) * Hq + g * G + h) * D + lane * C::kEPL;
#pragma unroll
        for (int e = 0; e < C::kEPL; e += 2) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(qh + e);
            qr[h][e] = bf16_lo(w) * scale_log2;
            qr[h][e + 1] = bf16_hi(w) * scale_log2;
        }
    }

    // P.V ownership: thread -> bf16 pair `pi` of D, key subset `ks` (keys ks, ks+KS, ...)
    const int pi = tid % (D / 2);
    const int ks = tid / (D / 2);
    float o[G][2];
#pragma unroll
    for (int h = 0; h < G; ++h) o[h][0] = o[h][1] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;   // meaningful in warp `h` for head h < G
    bool ok = true;

    for (int li = 0; li < n_live; ++li) {
        const int st = li % C::kStages;
        const int sub = live_list[li];
        const int kk0 = key0 + sub * kSubKeys;
        const int rows = min(kSubKeys, S_ctx - kk0);
        ok = mbar_wait(&full[st], (li / C::kStages) & 1, abort_flag);
        if (!ok) break;
        const uint8_t* Ks = smem + C::kRingOff + st * C::kStageBytes;
        const uint8_t* Vs = Ks + C::kSubBytes;
        // ---- scores: warp w takes keys w, w+8, w+16, w+24
#pragma unroll
        for (int kq = 0; kq < kSubKeys / kWarps; ++kq) {
            const int kr = warp + kq * kWarps;
            float acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = 0.f;
            if (kr < rows) {
                const uint32_t* krow =
                    reinterpret_cast<const uint32_t*>(Ks + kr * C::kRowBytes + lane * C::kEPL * 2);
#pragma unroll
                for (int e = 0; e < C::kEPL; e += 2) {
                    const uint32_t w = krow[e / 2];
                    const float k0 = bf16_lo(w), k1 = bf16_hi(w);
#pragma unroll
                    for (int h = 0; h < G; ++h) acc[h] = fmaf(qr[h][e + 1], k1, fmaf(qr[h][e], k0, acc[h]));
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = warp_sum(acc[h]);
            if (lane == 0) {
                const float mv = s_mask[sub * kSubKeys + kr];
#pragma unroll
                for (int h = 0; h < G; ++h)
                    s_score[h * kSubKeys + kr] = (kr < rows && mv != -INFINITY) ? acc[h] + mv : -INFINITY;
            }
        }
        __syncthreads();
        // the stage used two sub-tiles ago is free now: refill it
        if (tid == 0 && li >= 1 && li - 1 + C::kStages < n_live) issue(li - 1 + C::kStages);
        // ---- online softmax update: warp h owns head h, lane = key
        if (warp < G) {
            const float x = s_score[warp * kSubKeys + lane];
            const float m_new = fmaxf(m_run, warp_max(x));
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float p = ex2_approx(x - m_use);
            const float alpha = ex2_approx(m_run - m_use);
            l_run = l_run * alpha + warp_sum(p);
            m_run = m_new;
            s_score[warp * kSubKeys + lane] = p;
            if (lane == 0) s_alpha[warp] = alpha;
        }
        __syncthreads();
        // ---- O = alpha * O + P V over this thread's key subset
        const uint32_t* vcol = reinterpret_cast<const uint32_t*>(Vs) + pi;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a = s_alpha[h];
            o[h][0] *= a;
            o[h][1] *= a;
        }
#pragma unroll 4
        for (int kr = ks; kr < kSubKeys; kr += C::kKS) {
            if (kr >= rows) break;
            const uint32_t w = vcol[kr * (D / 2)];
            const float v0 = bf16_lo(w), v1 = bf16_hi(w);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = s_score[h * kSubKeys + kr];
                o[h][0] = fmaf(p, v0, o[h][0]);
                o[h][1] = fmaf(p, v1, o[h][1]);
            }
        }
    }
    if (!ok && tid == 0) {
        for (int li = 0; li < n_live && li < C::kStages; ++li) mbar_wait_drain(&full[li % C::kStages], 0);
    }
    __syncthreads();
    // ---- reduce the key subsets and write the partial (o, m, l)
#pragma unroll
    for (int h = 0; h < G; ++h) {
        s_red[(ks * G + h) * D + 2 * pi] = o[h][0];
        s_red[(ks * G + h) * D + 2 * pi + 1] = o[h][1];
    }
    __syncthreads();
    const size_t row_base = (static_cast<size_t>(b) * Hq + g * G) * n_split + split;
    for (int idx = tid; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        float acc = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < C::kKS; ++s2) acc += s_red[(s2 * G + h) * D + d];
        ws_o[(row_base + static_cast<size_t>(h) * n_split) * D + d] = acc;
    }
    if (warp < G && lane == 0) {
        ws_m[row_base + static_cast<size_t>(warp) * n_split] = m_run;
        ws_l[row_base + static_cast<size_t>(warp) * n_split] = l_run;
    }
}

// out[b,h] = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i   (m in log2 units)
template <int D>
__global__ void __launch_bounds__(D / 4)
decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_m,
                      const float* __restrict__ ws_l, uint16_t* __restrict__ out, int n_split) {
    const size_t row = blockIdx.x;   // b * Hq + h
    const float* m = ws_m + row * n_split;
    const float* l = ws_l + row * n_split;
    float M = -INFINITY;
    for (int i = 0; i < n_split; ++i) M = fmaxf(M, m[i]);
    const int d = threadIdx.x * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M != -INFINITY) {
        for (int i = 0; i < n_split; ++i) {
            if (m[i] == -INFINITY) continue;
            const float w = ex2_approx(m[i] - M);
            den = fmaf(w, l[i], den);
            const float4 oi = *reinterpret_cast<const float4*>(ws_o + (row * n_split + i) * D + d);
            acc.x = fmaf(w, oi.x, acc.x);
            acc.y = fmaf(w, oi.y, acc.y);
            acc.z = fmaf(w, oi.z, acc.z);
            acc.w = fmaf(w, oi.w, acc.w);
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(out + row * D + d) = pk;
}

template <int D, int G>
int launch_dg(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
              uint16_t* out, int B, int Hkv, int S_ctx, float scale, float* ws_o, float* ws_m,
              float* ws_l, cudaStream_t stream) {
    using C = Cfg<D>;
    static std::atomic<uint64_t> smem_done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -6;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(smem_done.load() & bit)) {
        if (cudaFuncSetAttribute(decode_split_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
            cudaSuccess)
            return -6;
        smem_done.fetch_or(bit);
    }
    const int n_split = num_splits(S_ctx);
    dim3 grid(n_split, Hkv, B);
    decode_split_kernel<D, G><<<grid, kThreads, C::kSmemBytes, stream>>>(
        q, k, v, mask, ws_o, ws_m, ws_l, Hkv, S_ctx, scale * kLog2e);
    decode_combine_kernel<D><<<B * Hkv * G, D / 4, 0, stream>>>(ws_o, ws_m, ws_l, out, n_split);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

template <int D>
int launch_d(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
             uint16_t* out, int B, int Hkv, int G, int S_ctx, float scale, float* ws_o,
             float* ws_m, float* ws_l, cudaStream_t s) {
    switch (G) {
        case 1: return launch_dg<D, 1>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 2: return launch_dg<D, 2>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 4: return launch_dg<D, 4>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 8: return launch_dg<D, 8>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        default: return -3;   // ATTN_ERR_UNSUPPORTED
    }
}

// Carves the workspace and launches split + combine on `stream`.
inline int launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
                  uint16_t* out, int B, int Hq, int Hkv, int G, int S_ctx, int D, float scale,
                  void* workspace, cudaStream_t stream) {
    const size_t rows = static_cast<size_t>(B) * Hq * num_splits(S_ctx);
    float* ws_o = static_cast<float*>(workspace);
    uint8_t* p = reinterpret_cast<uint8_t*>(ws_o + rows * D);
    const size_t ml = ((rows * sizeof(float) + 255) / 256) * 256;
    float* ws_m = reinterpret_cast<float*>(p);
    float* ws_l = reinterpret_cast<float*>(p + ml);
    switch (D) {
        case 128: return launch_d<128>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws_o, ws_m, ws_l, stream);
        case 256: return launch_d<256>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws_o, ws_m, ws_l, stream);
        case 512: return launch_d<512>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws_o, ws_m, ws_l, stream);
        default: return -3;
    }
}

}  // namespace dec
}  // namespace attn
