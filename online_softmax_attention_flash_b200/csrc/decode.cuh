// decode.cuh -- single-token GQA flash-decode for sm_100a.
//
// What it computes ("head_dim>128 (256/512) GQA Flash-Decode NKI Kernel for
// AWS Trainium", "Input contract"): for every batch entry b and query head h,
//   out[b,h] = softmax(scale * q[b,h] K[b,g]^T + attn_mask[b]) V[b,g],
//   g = h / num_kv_groups, S_q = 1, head_dim D in {128, 256, 512}.
//
// How. Decode is bound by HBM bandwidth (each K/V byte serves only
// num_kv_groups query heads), so the tensor cores stay idle and the design is
// about streaming K/V once, at full bandwidth, with little on-chip overhead:
//   * split-KV (the page's "multi-program dispatch" follow-on): grid =
//     (key splits, kv heads, batch); a CTA owns kSplitKeys keys of one (b, g)
//     and serves all num_kv_groups query heads of that kv head from the same
//     bytes (the pages' GQA head packing, as data reuse);
//   * inside the CTA every warp runs its own flash-decoding stream: it takes
//     every 4th live 8-key sub-tile, pulls K and V rows with bulk async copies
//     (cp.async.bulk) into a private shared-memory ring, and keeps its own
//     running max / sum / numerator, so the main loop has no CTA-wide barrier;
//   * q . k partial sums (lanes split D) are reduced with a transposed
//     butterfly: 8 keys x G heads values per lane are halved at every shuffle
//     step, one shuffle per (key, head) pair instead of five;
//   * 8-key sub-tiles whose mask is all -inf, or that lie past S_ctx, are never
//     read (length-aware skipping);
//   * at the end the four warps' states are merged in shared memory and one
//     unnormalised partial (o, m, l) per CTA goes to the workspace; a second
//     kernel combines the splits with the log-sum-exp rule.
// Scores are kept in log2 units (scale * log2 e folded into q) so every
// exponential is one ex2 instruction.
#pragma once

#include "ptx.cuh"
#include "tmap.cuh"

namespace attn {
namespace dec {

constexpr int kSubKeys = 8;                  // keys per sub-tile (one ring stage)
constexpr int kSplitKeys = 512;              // keys per CTA
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
    // warps per CTA and ring stages per warp: ~96 KB of ring per CTA (two CTAs per SM)
    // for D <= 256; D = 512 uses 4 warps x 2 stages (128 KB, one CTA per SM)
    static constexpr int kWarps = (D == 512) ? 4 : 6;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRowBytes = D * 2;
    static constexpr int kSubBytes = kSubKeys * kRowBytes;       // K (or V) rows of one sub-tile
    static constexpr int kStageBytes = 2 * kSubBytes;            // K then V
    static constexpr int kStages = (D == 128) ? 4 : 2;   // per warp
    static constexpr int kEPL = D / 32;                           // elements of D per lane
    static constexpr int kRingOff = 0;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kMaskOff = kRingOff + kRingBytes;                  // [kSplitKeys] fp32
    static constexpr int kScrOff = kMaskOff + kSplitKeys * 4;               // per warp: P [G][8], alpha [G]
    static constexpr int kScrFloats = kMaxGroups * kSubKeys + kMaxGroups;
    static constexpr int kListOff = kScrOff + kWarps * kScrFloats * 4;      // live sub-tiles
    static constexpr int kBarOff = kListOff + (kSubTiles + 4) * 4;
    static constexpr int kMiscOff = kBarOff + kWarps * kStages * 2 * 8;   // K and V barrier per stage
    static constexpr int kSmemBytes = kMiscOff + 16;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// EPL consecutive bf16 (EPL = 4, 8 or 16) as EPL / 2 packed words (8- or 16-byte loads).
template <int EPL>
__device__ __forceinline__ void load_bf16_words(const void* p, uint32_t (&w)[EPL / 2]) {
    if constexpr (EPL == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(p);
        w[0] = t.x;
        w[1] = t.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL / 8; ++i) {
            const uint4 t = reinterpret_cast<const uint4*>(p)[i];
            w[4 * i] = t.x;
            w[4 * i + 1] = t.y;
            w[4 * i + 2] = t.z;
            w[4 * i + 3] = t.w;
        }
    }
}

// Transposed butterfly: v[0..N) are per-lane partial sums of N different dot
// products; after the call lane L holds the full sum of value index
// idx(L) = L / (32 / N) in v[0] (N = 8, 16 or 32).
template <int N>
__device__ __forceinline__ void transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16, n = N; n > 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    // the 32 / N lanes that now share one value index differ in their low bits
#pragma unroll
    for (int o = (32 / N) / 2; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
}

template <int D, int G>
__global__ void __launch_bounds__(Cfg<D>::kThreads)
decode_split_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, const float* __restrict__ mask,
                    float* __restrict__ ws_o, float* __restrict__ ws_m, float* __restrict__ ws_l,
                    int Hkv, int S_ctx, float scale_log2) {
    using C = Cfg<D>;
    constexpr int kWarps = C::kWarps;
    constexpr int kThreads = C::kThreads;
    constexpr int kHeadsPerPass = G < 4 ? G : 4;       // N = 8 * heads <= 32 values per butterfly
    constexpr int kPasses = G / kHeadsPerPass;
    constexpr int kN = kSubKeys * kHeadsPerPass;
    constexpr int kBase = 32 / kN;                      // lanes sharing one value index
    extern __shared__ __align__(128) uint8_t smem[];
    float* s_mask = reinterpret_cast<float*>(smem + C::kMaskOff);
    int* live = reinterpret_cast<int*>(smem + C::kListOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);
    int* n_live_sm = reinterpret_cast<int*>(smem + C::kMiscOff + 4);

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hq = Hkv * G;
    const int n_split = gridDim.x;
    const int key0 = split * kSplitKeys;
    const size_t kv_base = (static_cast<size_t>(b) * Hkv + g) * S_ctx;
    float* scr = reinterpret_cast<float*>(smem + C::kScrOff) + warp * C::kScrFloats;
    uint64_t* my_full = full + warp * C::kStages * 2;   // [stage][K, V]
    uint8_t* my_ring = smem + C::kRingOff + warp * C::kStages * C::kStageBytes;

    // the combine kernel may be scheduled now; it waits for this grid's completion itself
    pdl_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < kWarps * C::kStages * 2; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // the previous kernel on the stream may still be reading this workspace: wait for it
    pdl_wait_predecessor();
    // additive mask of this split in log2 units (-inf past S_ctx); live 8-key sub-tiles
    for (int i = tid; i < kSplitKeys; i += kThreads) {
        const int key = key0 + i;
        float mv = -INFINITY;
        if (key < S_ctx) mv = mask ? mask[static_cast<size_t>(b) * S_ctx + key] * kLog2e : 0.f;
        s_mask[i] = mv;
    }
    __syncthreads();
    if (warp == 0) {
        int n = 0;
        for (int base = 0; base < kSubTiles; base += 32) {
            const int st = base + lane;
            bool any = false;
            if (st < kSubTiles)
#pragma unroll
                for (int kk = 0; kk < kSubKeys; ++kk) any |= (s_mask[st * kSubKeys + kk] != -INFINITY);
            const uint32_t bal = __ballot_sync(0xffffffffu, any);
            if (any) live[n + __popc(bal & ((1u << lane) - 1u))] = st;
            n += __popc(bal);
        }
        if (lane == 0) *n_live_sm = n;
    }
    __syncthreads();
    const int n_live = *n_live_sm;
    // this warp's share: live sub-tiles warp, warp + 4, ...
    const int my_count = n_live > warp ? (n_live - warp + kWarps - 1) / kWarps : 0;

    // K and V rows of this warp's i-th sub-tile go to stage i % kStages, each half with
    // its own barrier, so that K can be refilled as soon as the scores are computed
    int issued[2] = {0, 0};   // sub-tiles whose K / V copy this warp has started (lane 0)
    auto issue_half = [&](int i, int which) {
        issued[which] = i + 1;
        const int st = i % C::kStages;
        const int sub = live[warp + i * kWarps];
        const int kk0 = key0 + sub * kSubKeys;
        const int rows = min(kSubKeys, S_ctx - kk0);
        const uint32_t bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
        uint8_t* dst = my_ring + st * C::kStageBytes + which * C::kSubBytes;
        mbar_arrive_expect_tx(&my_full[2 * st + which], bytes);
        bulk_load(dst, (which ? v : k) + (kv_base + kk0) * D, bytes, &my_full[2 * st + which]);
    };
    if (lane == 0)
        for (int i = 0; i < my_count && i < C::kStages; ++i) {
            issue_half(i, 0);
            issue_half(i, 1);
        }

    // q of the G heads: this lane's slice [lane*EPL, lane*EPL + EPL), pre-scaled to log2 units
    float qr[G][C::kEPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint16_t* qh = q + (static_cast<size_t>(b) * Hq + g * G + h) * D + lane * C::kEPL;
        uint32_t ws[C::kEPL / 2];
        load_bf16_words<C::kEPL>(qh, ws);
#pragma unroll
        for (int i = 0; i < C::kEPL / 2; ++i) {
            qr[h][2 * i] = bf16_lo(ws[i]) * scale_log2;
            qr[h][2 * i + 1] = bf16_hi(ws[i]) * scale_log2;
        }
    }
    float o[G][C::kEPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < C::kEPL; ++e) o[h][e] = 0.f;
    float m_run[G], l_run[G];   // per head (meaningful on every lane)
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
    }
    bool ok = true;

    for (int i = 0; i < my_count; ++i) {
        const int st = i % C::kStages;
        const int sub = live[warp + i * kWarps];
        const int kk0 = key0 + sub * kSubKeys;
        const int rows = min(kSubKeys, S_ctx - kk0);
        ok = mbar_wait(&my_full[2 * st], (i / C::kStages) & 1, abort_flag);
        if (!ok) break;
        const uint8_t* Ks = my_ring + st * C::kStageBytes;
        const uint8_t* Vs = Ks + C::kSubBytes;
#pragma unroll
        for (int pass = 0; pass < kPasses; ++pass) {
            // ---- scores of 8 keys x kHeadsPerPass heads: lane-split dot products, then butterfly
            float part[32];
#pragma unroll
            for (int kk = 0; kk < kSubKeys; ++kk) {
                float2 acc[kHeadsPerPass];   // even / odd elements, packed fp32x2 FMAs
#pragma unroll
                for (int hh = 0; hh < kHeadsPerPass; ++hh) acc[hh] = make_float2(0.f, 0.f);
                uint32_t ws[C::kEPL / 2];
                load_bf16_words<C::kEPL>(Ks + kk * C::kRowBytes + lane * C::kEPL * 2, ws);
#pragma unroll
                for (int i2 = 0; i2 < C::kEPL / 2; ++i2) {
                    const float2 kv = make_float2(bf16_lo(ws[i2]), bf16_hi(ws[i2]));
#pragma unroll
                    for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                        const int h = pass * kHeadsPerPass + hh;
                        acc[hh] = __ffma2_rn(make_float2(qr[h][2 * i2], qr[h][2 * i2 + 1]), kv, acc[hh]);
                    }
                }
#pragma unroll
                for (int hh = 0; hh < kHeadsPerPass; ++hh) part[hh * kSubKeys + kk] = acc[hh].x + acc[hh].y;
            }
            transpose_reduce<kN>(part, lane);
            if (pass == kPasses - 1) {   // every lane is done reading K of this stage
                __syncwarp();
                if (lane == 0 && i + C::kStages < my_count) issue_half(i + C::kStages, 0);
            }
            // lane now holds the score of value idx = lane / kBase: head hh = idx / 8, key kk = idx % 8
            const int idx = lane / kBase;
            const int hh_me = idx / kSubKeys, kk_me = idx % kSubKeys;
            const float mv = s_mask[sub * kSubKeys + kk_me];
            float x = (kk_me < rows && mv != -INFINITY) ? part[0] + mv : -INFINITY;
            // ---- online softmax per head over its 8 keys (lanes of one head form a group)
            float mt = x;
#pragma unroll
            for (int off = kBase; off < kBase * kSubKeys; off <<= 1)
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            // running max of this lane's head (unrolled select keeps m_run in registers)
            float m_old = -INFINITY;
#pragma unroll
            for (int hh = 0; hh < kHeadsPerPass; ++hh)
                if (hh_me == hh) m_old = m_run[pass * kHeadsPerPass + hh];
            const float m_new = fmaxf(m_old, mt);
            const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
            const float p = ex2_approx(x - m_use);
            const float alpha = ex2_approx(m_old - m_use);
            float ps = p;
#pragma unroll
            for (int off = kBase; off < kBase * kSubKeys; off <<= 1)
                ps += __shfl_xor_sync(0xffffffffu, ps, off);
            // publish P and alpha of this pass for the P.V step
            if ((lane % kBase) == 0) scr[hh_me * kSubKeys + kk_me] = p;
            if ((lane % kBase) == 0 && kk_me == 0) scr[kMaxGroups * kSubKeys + hh_me] = alpha;
            __syncwarp();
            // every lane updates the running state of the heads of this pass; O is rescaled
            // only if some head's max moved (after the first sub-tiles it rarely does)
            const bool any_moved = __any_sync(0xffffffffu, m_new != m_old);
#pragma unroll
            for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                const int h = pass * kHeadsPerPass + hh;
                const float a = scr[kMaxGroups * kSubKeys + hh];
                const float mn = __shfl_sync(0xffffffffu, m_new, hh * kSubKeys * kBase);
                const float sum = __shfl_sync(0xffffffffu, ps, hh * kSubKeys * kBase);
                l_run[h] = l_run[h] * a + sum;
                m_run[h] = mn;
                if (any_moved) {
#pragma unroll
                    for (int e = 0; e < C::kEPL; e += 2) {
                        const float2 r = __fmul2_rn(make_float2(o[h][e], o[h][e + 1]), make_float2(a, a));
                        o[h][e] = r.x;
                        o[h][e + 1] = r.y;
                    }
                }
            }
            if (pass == 0) {
                if (!mbar_wait(&my_full[2 * st + 1], (i / C::kStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
            }
            // ---- O += P V for this pass's heads (rows past S_ctx hold stale data: skipped)
#pragma unroll
            for (int kk = 0; kk < kSubKeys; ++kk) {
                if (kk < rows) {
                    uint32_t ws[C::kEPL / 2];
                    load_bf16_words<C::kEPL>(Vs + kk * C::kRowBytes + lane * C::kEPL * 2, ws);
                    float pk[kHeadsPerPass];
#pragma unroll
                    for (int hh = 0; hh < kHeadsPerPass; ++hh) pk[hh] = scr[hh * kSubKeys + kk];
#pragma unroll
                    for (int i2 = 0; i2 < C::kEPL / 2; ++i2) {
                        const float2 vv = make_float2(bf16_lo(ws[i2]), bf16_hi(ws[i2]));
#pragma unroll
                        for (int hh = 0; hh < kHeadsPerPass; ++hh) {
                            const int h = pass * kHeadsPerPass + hh;
                            const float2 r = __ffma2_rn(make_float2(pk[hh], pk[hh]), vv,
                                                        make_float2(o[h][2 * i2], o[h][2 * i2 + 1]));
                            o[h][2 * i2] = r.x;
                            o[h][2 * i2 + 1] = r.y;
                        }
                    }
                }
            }
            __syncwarp();   // scratch is rewritten by the next pass / sub-tile
        }
        if (!ok) break;
        // V of this stage is consumed: refill it with the sub-tile kStages ahead
        if (lane == 0 && i + C::kStages < my_count) issue_half(i + C::kStages, 1);
    }
    if (!ok && lane == 0) {   // let every copy this warp started land before the CTA exits
        for (int which = 0; which < 2; ++which)
            for (int i = max(0, issued[which] - C::kStages); i < issued[which]; ++i)
                mbar_wait_drain(&my_full[2 * (i % C::kStages) + which], (i / C::kStages) & 1);
    }
    __syncthreads();   // every warp is done with its ring: reuse it for the merge

    // ---- merge the four warps' states; write one unnormalised partial per (head, split)
    float* mo = reinterpret_cast<float*>(smem + C::kRingOff);            // [warp][G][D]
    float* mm = mo + kWarps * G * D;                                        // [warp][G]
    float* ml = mm + kWarps * G;                                            // [warp][G]
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < C::kEPL; ++e) mo[(warp * G + h) * D + lane * C::kEPL + e] = o[h][e];
    if (lane == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            mm[warp * G + h] = m_run[h];
            ml[warp * G + h] = l_run[h];
        }
    __syncthreads();
    const size_t row_base = (static_cast<size_t>(b) * Hq + g * G) * n_split + split;
    for (int idx = tid; idx < G * D; idx += kThreads) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * G + h]);
        float acc = 0.f, lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float mw = mm[w * G + h];
                if (mw == -INFINITY) continue;
                const float f = ex2_approx(mw - M);
                acc = fmaf(f, mo[(w * G + h) * D + d], acc);
                lsum = fmaf(f, ml[w * G + h], lsum);
            }
        }
        ws_o[(row_base + static_cast<size_t>(h) * n_split) * D + d] = acc;
        if (d == 0) {
            ws_m[row_base + static_cast<size_t>(h) * n_split] = M;
            ws_l[row_base + static_cast<size_t>(h) * n_split] = lsum;
        }
    }
}

// out[b,h] = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i   (m in log2 units)
template <int D>
__global__ void __launch_bounds__(D / 4)
decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_m,
                      const float* __restrict__ ws_l, uint16_t* __restrict__ out, int n_split) {
    // launched as a programmatic dependent of the split kernel: wait until its writes
    // to the workspace are complete and visible
    pdl_wait_predecessor();
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
    static_assert(C::kRingBytes >= C::kWarps * G * (D + 2) * 4, "merge area must fit in the ring");
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
    if (launch_pdl(decode_split_kernel<D, G>, grid, dim3(C::kThreads), C::kSmemBytes, stream, q, k,
                   v, mask, ws_o, ws_m, ws_l, Hkv, S_ctx, scale * kLog2e))
        return -6;
    return launch_pdl(decode_combine_kernel<D>, dim3(B * Hkv * G), dim3(D / 4), 0, stream,
                      static_cast<const float*>(ws_o), static_cast<const float*>(ws_m),
                      static_cast<const float*>(ws_l), out, n_split);
}

template <int D>
int launch_d(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
             uint16_t* out, int B, int Hkv, int G, int S_ctx, float scale, float* ws_o,
             float* ws_m, float* ws_l, cudaStream_t s) {
    switch (G) {
        case 1: return launch_dg<D, 1>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 2: return launch_dg<D, 2>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 4: return launch_dg<D, 4>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
        case 8:
            if constexpr (D <= 256)
                return launch_dg<D, 8>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws_o, ws_m, ws_l, s);
            return -3;   // ATTN_ERR_UNSUPPORTED: D = 512 with 8 heads per group
        default: return -3;
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
