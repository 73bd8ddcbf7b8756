// proj.cuh -- the projections on either side of the attention core, for sm_100a.
//
// What they compute ("V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2",
// "Repository layout": the attention block is QKV projection + RoPE, the
// attention inner, and the output projection; "vit-encoder-neuron-kernels",
// "Kernels": both RoPE lane pairings):
//   qkv: t = x W_qkv^T + b_qkv for x [B, S, C] bf16, W_qkv [3 H D, C] bf16; the
//        three column blocks of t are Q, K, V, column h D + d of a block is head h,
//        lane d; Q and K are rotated (RoPE, [S, D/2] cos / sin tables) and all
//        three are written as bf16 in the attention layout [B, H, S, D];
//   out: y = a W_o^T + b_o with a[b, s, h D + d] = o[b, h, s, d] (the attention
//        output, bf16) and W_o [C_out, H D] bf16; y [B, S, C_out] fp32.
//
// How. One GEMM kernel for both: a CTA owns a tile of 128 tokens of one batch entry
// by BN output columns. A TMA producer warp streams 64-wide K chunks of the
// activation tile (x as [B][S][C], or o through a rank-4 map [B][H][S][D] whose
// K chunk selects head and lane range, so the heads are gathered side by side
// without a copy) and of the weight tile through a 4-6 stage ring; one thread of
// the MMA warp issues tcgen05.mma (M = 128, N = BN, bf16 operands, fp32
// accumulate in TMEM); four epilogue warps (one TMEM lane = one token each) read
// the accumulator, add the bias and, for Q and K, rotate lane pairs before the
// bf16 rounding, so the rotated Q / K never make a separate pass through HBM.
#pragma once

#include "ptx.cuh"
#include "tmap.cuh"

namespace attn {
namespace proj {

constexpr int kBM = 128;                 // tokens per tile = TMEM lanes
constexpr int kBK = 64;                  // K chunk: 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;            // warps 0-3 epilogue, 4 producer, 5 MMA issuer
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kABytes = kBM * 128;

template <int BN>
struct Cfg {
    static constexpr int kBBytes = BN * 128;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (BN == 256) ? 4 : 6;
    static constexpr int kBarOff = kStages * kStageBytes;
    // full[S], empty[S], acc_full[2], acc_empty[2], mma_done, bias_ready[2]
    static constexpr int kNumBars = 2 * kStages + 7;
    static constexpr int kBiasOff = kBarOff + kNumBars * 8 + 8;   // [2][BN] fp32 tile biases
    static constexpr int kMiscOff = kBiasOff + 2 * BN * 4;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr uint32_t kTmemCols = 2 * BN;                // two accumulators
};

struct Params {
    int S, K;                 // tokens per batch entry; reduction length (C, or H * D)
    int H, D;                 // heads and head dim (qkv: of the outputs; out: of the input o)
    const float* bias;        // [N] fp32 or nullptr
    // qkv
    uint16_t* q;
    uint16_t* k;
    uint16_t* v;
    const float* cos_t;       // [S, D/2] or nullptr
    const float* sin_t;
    int rope;                 // 0 none, 1 half (j, j + D/2), 2 interleaved (2j, 2j + 1)
    // out
    float* y;
    int n_out;                // C_out
    // tiles: m_tiles x n_tiles x B, n fastest
    int m_tiles, n_tiles, n_total;
};

__device__ __forceinline__ float4 ldg4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }

// 16 consecutive accumulator columns of this thread's row, plus bias.
__device__ __forceinline__ void acc16(uint32_t taddr, const float* bias, float (&x)[16]) {
    uint32_t u[16];
    tmem_ld16_wait(taddr, u);
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(u[i]);
    if (bias) {
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
            const float4 b4 = ldg4(bias + i);
            x[i] += b4.x;
            x[i + 1] += b4.y;
            x[i + 2] += b4.z;
            x[i + 3] += b4.w;
        }
    }
}

__device__ __forceinline__ void store_bf16x16(uint16_t* dst, const float (&x)[16]) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    d4[0] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                       pack_bf16x2(x[6], x[7]));
    d4[1] = make_uint4(pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]),
                       pack_bf16x2(x[12], x[13]), pack_bf16x2(x[14], x[15]));
}

template <int BN, bool kOut, int kD>
__global__ void __launch_bounds__(kThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const Params p) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;   // [2]
    uint64_t* acc_empty = acc_full + 2;         // [2]
    uint64_t* mma_done = acc_empty + 2;
    uint64_t* bias_ready = mma_done + 1;        // [2]: the tile's biases are staged
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int n_k = p.K / kBK;
    // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ... (persistent)
    const int my_tiles = p.n_total > static_cast<int>(blockIdx.x)
                             ? (p.n_total - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                             : 0;
    auto tile_coords = [&](int i, int& s0, int& n0, int& b) {
        const int t = blockIdx.x + i * gridDim.x;
        n0 = (t % p.n_tiles) * BN;
        s0 = ((t / p.n_tiles) % p.m_tiles) * kBM;
        b = t / (p.n_tiles * p.m_tiles);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);   // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        mbar_init(&bias_ready[0], 128);
        mbar_init(&bias_ready[1], 128);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane_id() == 0) {
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_b);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait_predecessor();
    int issued = 0;   // producer: K chunks (over all of this CTA's tiles) whose copies were started

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane_id() == 0) {
            bool ok = true;
            for (int i = 0; i < my_tiles && ok; ++i) {
                int s0, n0, b;
                tile_coords(i, s0, n0, b);
                for (int kc = 0; kc < n_k; ++kc) {
                    const int g = issued;   // chunk number over the whole ring
                    const int st = g % C::kStages;
                    const uint32_t use = g / C::kStages;
                    if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a_dst = smem + st * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[st], C::kStageBytes);
                    if constexpr (kOut) {
                        const int kk = kc * kBK;   // column h D + d0 of the side-by-side heads
                        tma_load_4d(a_dst, &tm_a, &full[st], kk % kD, s0, kk / kD, b);
                    } else {
                        tma_load_3d(a_dst, &tm_a, &full[st], kc * kBK, s0, b);
                    }
                    tma_load_2d(a_dst + kABytes, &tm_b, &full[st], kc * kBK, n0);
                    issued = g + 1;
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane_id() == 0) {
            constexpr uint32_t idesc = make_idesc(kBM, BN, 1, 1, 0, 0);   // bf16 x bf16, both K-major
            const uint64_t da = smem_desc(smem_u32(smem), 16, 1024);
            const uint64_t db = smem_desc(smem_u32(smem + kABytes), 16, 1024);
            bool ok = true;
            int g = 0;
            for (int i = 0; i < my_tiles && ok; ++i) {
                const int acc = i & 1;
                // the epilogue has read this accumulator's previous tile
                if (i >= 2 && !mbar_wait(&acc_empty[acc], ((i >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kc = 0; kc < n_k; ++kc, ++g) {
                    const int st = g % C::kStages;
                    if (!mbar_wait(&full[st], (g / C::kStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t so = static_cast<uint64_t>((st * C::kStageBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)   // K-steps of 16 = 32 bytes along the row
                        mma_f16_ss(d_tmem, da + so + 2 * kk, db + so + 2 * kk, idesc,
                                   (kc > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[st]);
                }
                if (ok) tc_commit(&acc_full[acc]);
            }
            tc_commit(mma_done);   // every MMA of this CTA (teardown waits for it on an abort)
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (4 warps)
        const int r = threadIdx.x;   // row of the tile = TMEM lane
        float* sbias_all = reinterpret_cast<float*>(smem + C::kBiasOff);
        constexpr int kHalf = kD / 2;
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        for (int i = 0; i < my_tiles; ++i) {
            int s0, n0, b;
            tile_coords(i, s0, n0, b);
            const int acc = i & 1;
            const int row = s0 + r;
            const bool valid = row < p.S;
            // Stage what the epilogue needs besides the accumulator while the K loop of this
            // tile runs: the tile's BN biases (shared memory, read by every row) and this row's
            // RoPE cos / sin (registers; the same for every head of the tile).
            float* sbias = sbias_all + acc * BN;
            for (int c = r; c < BN; c += 128) sbias[c] = p.bias ? __ldg(p.bias + n0 + c) : 0.f;
            float co[kOut ? 1 : kHalf], si[kOut ? 1 : kHalf];
            bool rot = false;
            uint16_t* dst_t = nullptr;
            int h0 = 0;
            if constexpr (!kOut) {
                const int HD = p.H * kD;
                const int which = n0 / HD;              // 0 q, 1 k, 2 v (a tile never straddles)
                dst_t = which == 0 ? p.q : (which == 1 ? p.k : p.v);
                rot = which < 2 && p.rope != 0;
                h0 = (n0 % HD) / kD;
                if (rot && valid) {
                    const float* cs = p.cos_t + static_cast<size_t>(row) * kHalf;
                    const float* sn = p.sin_t + static_cast<size_t>(row) * kHalf;
#pragma unroll
                    for (int j = 0; j < kHalf; j += 4) {
                        const float4 c4 = ldg4(cs + j), s4 = ldg4(sn + j);
                        co[j] = c4.x; co[j + 1] = c4.y; co[j + 2] = c4.z; co[j + 3] = c4.w;
                        si[j] = s4.x; si[j + 1] = s4.y; si[j + 2] = s4.z; si[j + 3] = s4.w;
                    }
                }
            }
            // Once all 128 threads have arrived the biases are visible to the four warps; a
            // warp also arrives only after it finished tile i - 1, so the next write to this
            // buffer (tile i + 2, after this wait) cannot overtake a reader of tile i. An
            // mbarrier, not bar.sync: a warp that gave up must not leave the others waiting.
            mbar_arrive(&bias_ready[acc]);
            if (!mbar_wait_warp(&bias_ready[acc], (i >> 1) & 1, abort_flag)) break;
            if (!mbar_wait_warp(&acc_full[acc], (i >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t t_row = t_lane + acc * BN;
            if constexpr (kOut) {
                float* yrow = p.y + (static_cast<size_t>(b) * p.S + row) * p.n_out + n0;
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t u[32];
                    tmem_ld32_wait(t_row + c, u);
                    if (valid) {
                        float4* d4 = reinterpret_cast<float4*>(yrow + c);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            d4[q4] = make_float4(__uint_as_float(u[4 * q4]) + sbias[c + 4 * q4],
                                                 __uint_as_float(u[4 * q4 + 1]) + sbias[c + 4 * q4 + 1],
                                                 __uint_as_float(u[4 * q4 + 2]) + sbias[c + 4 * q4 + 2],
                                                 __uint_as_float(u[4 * q4 + 3]) + sbias[c + 4 * q4 + 3]);
                    }
                }
            } else {
#pragma unroll 1
                for (int hh = 0; hh < BN / kD; ++hh) {
                    const int c0 = hh * kD;             // first tile column of this head
                    uint16_t* orow = dst_t + ((static_cast<size_t>(b) * p.H + h0 + hh) * p.S + row) * kD;
                    if (kD == 128 && rot && p.rope == 1) {
                        // rotate-half at kD = 128: lanes j and j + 64, 16 pairs at a time
#pragma unroll
                        for (int j0 = 0; j0 < kHalf; j0 += 16) {
                            uint32_t ua[16], ub[16];
                            tmem_ld16_wait(t_row + c0 + j0, ua);
                            tmem_ld16_wait(t_row + c0 + kHalf + j0, ub);
                            float xa[16], xb[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const float a = __uint_as_float(ua[e]) + sbias[c0 + j0 + e];
                                const float bb = __uint_as_float(ub[e]) + sbias[c0 + kHalf + j0 + e];
                                xa[e] = fmaf(a, co[j0 + e], -(bb * si[j0 + e]));
                                xb[e] = fmaf(a, si[j0 + e], bb * co[j0 + e]);
                            }
                            if (valid) {
                                store_bf16x16(orow + j0, xa);
                                store_bf16x16(orow + kHalf + j0, xb);
                            }
                        }
                        continue;
                    }
                    // the head's kD accumulator columns, 64 per TMEM load
#pragma unroll
                    for (int part = 0; part < kD / 64; ++part) {
                        float x[64];
                        {
                            uint32_t u[64];
                            tmem_ld64_wait(t_row + c0 + 64 * part, u);
#pragma unroll
                            for (int e = 0; e < 64; ++e) x[e] = __uint_as_float(u[e]) + sbias[c0 + 64 * part + e];
                        }
                        if (rot && p.rope == 2) {
                            // interleaved: lanes (2j, 2j + 1), j = 32 part .. 32 part + 31
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int j = 32 * part + e;
                                const float a0 = x[2 * e], a1 = x[2 * e + 1];
                                x[2 * e] = fmaf(a0, co[j], -(a1 * si[j]));
                                x[2 * e + 1] = fmaf(a0, si[j], a1 * co[j]);
                            }
                        } else if (rot && p.rope == 1) {
                            // rotate-half at kD = 64: lanes j and j + 32 in this part
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const float a = x[j], bb = x[j + 32];
                                x[j] = fmaf(a, co[j], -(bb * si[j]));
                                x[j + 32] = fmaf(a, si[j], bb * co[j]);
                            }
                        }
                        if (valid) {
                            uint4* d4 = reinterpret_cast<uint4*>(orow + 64 * part);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                d4[e] = make_uint4(pack_bf16x2(x[8 * e], x[8 * e + 1]), pack_bf16x2(x[8 * e + 2], x[8 * e + 3]),
                                                   pack_bf16x2(x[8 * e + 4], x[8 * e + 5]), pack_bf16x2(x[8 * e + 6], x[8 * e + 7]));
                        }
                    }
                }
            }
            // this accumulator may take the tile after next
            tc_fence_before();
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&acc_empty[acc]);
        }
        tc_wait_st();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // A bounded wait ran out somewhere: let every started copy land and every MMA
        // complete before this CTA frees TMEM and exits.
        if (warp == kProducerWarp && lane_id() == 0)
            for (int g = (issued > C::kStages ? issued - C::kStages : 0); g < issued; ++g)
                mbar_wait_drain(&full[g % C::kStages], (g / C::kStages) & 1);
        if (warp == kMmaWarp && lane_id() == 0) mbar_wait_drain(mma_done, 0);
        __syncwarp();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// Persistent grid: one CTA per SM (each holds ~200 KB of shared memory), at most one per tile.
inline int persistent_grid(int n_tiles, int* grid) {
    static std::atomic<int> sms_for_dev[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -6;
    int sms = sms_for_dev[dev].load();
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -6;
        sms_for_dev[dev].store(sms);
    }
    *grid = n_tiles < sms ? n_tiles : sms;
    return 0;
}

// Dynamic shared-memory opt-in once per (instantiation, device).
template <int BN, bool kOut, int kD>
inline int prepare() {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -6;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return 0;
    if (cudaFuncSetAttribute(proj_gemm_kernel<BN, kOut, kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<BN>::kSmemBytes) != cudaSuccess)
        return -6;
    done.fetch_or(bit);
    return 0;
}

// QKV projection (+ RoPE on Q, K): x [B, S, C], w [3 H D, C], outputs [B, H, S, D].
template <int BN, int kD>
inline int launch_qkv_t(const CUtensorMap& ta, const uint16_t* w, int C, int HD, const Params& p,
                        int B, cudaStream_t stream) {
    int rc;
    if ((rc = prepare<BN, false, kD>())) return rc;
    CUtensorMap tb;
    if ((rc = encode_map_2d_bf16(&tb, w, C, 3ull * HD, kBK, BN))) return rc;
    Params q = p;
    q.m_tiles = (p.S + kBM - 1) / kBM;
    q.n_tiles = 3 * HD / BN;
    q.n_total = q.m_tiles * q.n_tiles * B;
    int grid = 0;
    if ((rc = persistent_grid(q.n_total, &grid))) return rc;
    return launch_pdl(proj_gemm_kernel<BN, false, kD>, dim3(grid), dim3(kThreads), Cfg<BN>::kSmemBytes,
                      stream, ta, tb, q);
}

inline int launch_qkv(const uint16_t* x, const uint16_t* w, const float* bias, const float* cos_t,
                      const float* sin_t, int rope, int B, int S, int C, int H, int D, uint16_t* q,
                      uint16_t* k, uint16_t* v, cudaStream_t stream) {
    const int HD = H * D;
    Params p{};
    p.S = S;
    p.K = C;
    p.H = H;
    p.D = D;
    p.bias = bias;
    p.q = q;
    p.k = k;
    p.v = v;
    p.cos_t = cos_t;
    p.sin_t = sin_t;
    p.rope = rope;
    CUtensorMap ta;
    int rc;
    if ((rc = encode_map_3d_bf16(&ta, x, C, S, B, kBK, kBM))) return rc;
    if (HD % 256 == 0)
        return D == 64 ? launch_qkv_t<256, 64>(ta, w, C, HD, p, B, stream)
                       : launch_qkv_t<256, 128>(ta, w, C, HD, p, B, stream);
    return D == 64 ? launch_qkv_t<128, 64>(ta, w, C, HD, p, B, stream)
                   : launch_qkv_t<128, 128>(ta, w, C, HD, p, B, stream);
}

// Output projection: o [B, H, S, D] (heads side by side), w [C_out, H D] -> y [B, S, C_out] fp32.
template <int kD>
inline int launch_out_t(const uint16_t* o, const uint16_t* w, const Params& p, int B, int H,
                        cudaStream_t stream) {
    int rc;
    if ((rc = prepare<128, true, kD>())) return rc;
    CUtensorMap ta, tb;
    if ((rc = encode_map_4d_bf16(&ta, o, kD, p.S, H, B, kBK, kBM))) return rc;
    if ((rc = encode_map_2d_bf16(&tb, w, static_cast<uint64_t>(H) * kD, p.n_out, kBK, 128))) return rc;
    Params q = p;
    q.m_tiles = (p.S + kBM - 1) / kBM;
    q.n_tiles = p.n_out / 128;
    q.n_total = q.m_tiles * q.n_tiles * B;
    int grid = 0;
    if ((rc = persistent_grid(q.n_total, &grid))) return rc;
    return launch_pdl(proj_gemm_kernel<128, true, kD>, dim3(grid), dim3(kThreads), Cfg<128>::kSmemBytes,
                      stream, ta, tb, q);
}

inline int launch_out(const uint16_t* o, const uint16_t* w, const float* bias, int B, int S, int H,
                      int D, int C_out, float* y, cudaStream_t stream) {
    Params p{};
    p.S = S;
    p.K = H * D;
    p.H = H;
    p.D = D;
    p.bias = bias;
    p.y = y;
    p.n_out = C_out;
    return D == 64 ? launch_out_t<64>(o, w, p, B, H, stream) : launch_out_t<128>(o, w, p, B, H, stream);
}

}  // namespace proj
}  // namespace attn
