// rope.cuh -- rotary position embedding of Q and K rows for sm_100a.
//
// What it computes ("vit-encoder-neuron-kernels", section "Kernels": the encoder
// attention takes per-token rotation tables and supports two pairings of the
// head-dim lanes): for every row (b, h, s) of q and of k, [B, H, S, D] bf16, and
// every pair j = 0 .. D/2 - 1 with lanes (ia, ib) = (j, j + D/2) ("half":
// DINOv3, EVA-02, Llama) or (2j, 2j + 1) ("interleaved": V-JEPA2),
//     x'[ia] = x[ia] cos[s, j] - x[ib] sin[s, j]
//     x'[ib] = x[ia] sin[s, j] + x[ib] cos[s, j]
// in fp32, rounded to bf16 (round-to-nearest-even).
//
// How. The rotation is elementwise and HBM-bound (read Q and K, write them
// back; the [S, D/2] tables stay in L2 across heads), so it runs as its own
// pass rather than inside the attention kernel, whose softmax warps are its
// critical path: rotating K there would be repeated by every CTA of a head.
// One launch covers Q (blockIdx.y = 0) and K (blockIdx.y = 1); a thread rotates
// 8 pairs of one row with 16-byte vector loads and stores (32 bytes of the row,
// 8 cosines and 8 sines), grid-striding over the rows. In place is allowed
// (each thread writes exactly the bytes it read).
#pragma once

#include "ptx.cuh"
#include "tmap.cuh"

namespace attn {
namespace rope {

constexpr int kThreads = 256;
constexpr int kPairs = 8;   // pairs per thread

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <bool kInterleaved>
__global__ void __launch_bounds__(kThreads)
rope_qk_kernel(const uint16_t* q, const uint16_t* k, uint16_t* q_out, uint16_t* k_out,
               const float* __restrict__ cos_t, const float* __restrict__ sin_t, long long rows,
               int S, int D) {
    // Nothing is read before the previous kernel on the stream has finished (it may be
    // writing q or k); the next kernel may set up meanwhile.
    pdl_launch_dependents();
    pdl_wait_predecessor();
    const uint16_t* x = blockIdx.y ? k : q;
    uint16_t* y = blockIdx.y ? k_out : q_out;
    const int half = D / 2;
    const int groups = half / kPairs;
    const long long total = rows * groups;
    for (long long i = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * kThreads) {
        const long long row = i / groups;
        const int j0 = static_cast<int>(i - row * groups) * kPairs;
        const int s = static_cast<int>(row % S);
        const float4* cp = reinterpret_cast<const float4*>(cos_t + static_cast<size_t>(s) * half + j0);
        const float4* sp = reinterpret_cast<const float4*>(sin_t + static_cast<size_t>(s) * half + j0);
        const float4 c0 = __ldg(cp), c1 = __ldg(cp + 1), s0 = __ldg(sp), s1 = __ldg(sp + 1);
        const float c[kPairs] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sn[kPairs] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const uint16_t* xr = x + row * D;
        uint16_t* yr = y + row * D;
        if constexpr (kInterleaved) {
            // lanes 2 j0 .. 2 j0 + 15: word i holds the pair (2 (j0 + i), 2 (j0 + i) + 1)
            const uint4* src = reinterpret_cast<const uint4*>(xr + 2 * j0);
            const uint4 u0 = src[0], u1 = src[1];
            const uint32_t w[kPairs] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t o[kPairs];
#pragma unroll
            for (int p = 0; p < kPairs; ++p) {
                const float a = lo_bf16(w[p]), b = hi_bf16(w[p]);
                o[p] = pack_bf16x2(fmaf(a, c[p], -(b * sn[p])), fmaf(a, sn[p], b * c[p]));
            }
            uint4* dst = reinterpret_cast<uint4*>(yr + 2 * j0);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
            // lanes j0 .. j0 + 7 pair with lanes j0 + D/2 .. j0 + D/2 + 7
            const uint4 ua = *reinterpret_cast<const uint4*>(xr + j0);
            const uint4 ub = *reinterpret_cast<const uint4*>(xr + half + j0);
            const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
            const uint32_t wb[4] = {ub.x, ub.y, ub.z, ub.w};
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
                float ra[2], rb[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int p = 2 * w2 + e;
                    const float a = e ? hi_bf16(wa[w2]) : lo_bf16(wa[w2]);
                    const float b = e ? hi_bf16(wb[w2]) : lo_bf16(wb[w2]);
                    ra[e] = fmaf(a, c[p], -(b * sn[p]));
                    rb[e] = fmaf(a, sn[p], b * c[p]);
                }
                oa[w2] = pack_bf16x2(ra[0], ra[1]);
                ob[w2] = pack_bf16x2(rb[0], rb[1]);
            }
            *reinterpret_cast<uint4*>(yr + j0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
            *reinterpret_cast<uint4*>(yr + half + j0) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
        }
    }
}

// Rotates q and k (both [B, H, S, D]) into q_out and k_out on `stream`.
inline int launch(const uint16_t* q, const uint16_t* k, uint16_t* q_out, uint16_t* k_out,
                  const float* cos_t, const float* sin_t, int B, int H, int S, int D,
                  bool interleaved, cudaStream_t stream) {
    const long long rows = static_cast<long long>(B) * H * S;
    const long long work = rows * (D / 2 / kPairs);
    const long long want = (work + kThreads - 1) / kThreads;
    const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
    if (interleaved)
        return launch_pdl(rope_qk_kernel<true>, dim3(blocks, 2), dim3(kThreads), 0, stream, q, k,
                          q_out, k_out, cos_t, sin_t, rows, S, D);
    return launch_pdl(rope_qk_kernel<false>, dim3(blocks, 2), dim3(kThreads), 0, stream, q, k,
                      q_out, k_out, cos_t, sin_t, rows, S, D);
}

}  // namespace rope
}  // namespace attn
