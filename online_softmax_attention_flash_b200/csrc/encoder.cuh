// encoder.cuh -- non-causal multi-head encoder attention forward for sm_100a.
//
// What it computes: out[b,h] = softmax(scale * Q K^T + key_bias[b]) V for
// q/k/v/out in [B, H, S, D] bf16, D in {64, 128}: the attention core of the
// ViT / NewBERT encoder pages ("V-JEPA2 ViT-L Encoder NKI Kernels for AWS
// Trainium2", "vit-encoder-neuron-kernels": bidirectional self-attention with
// head_dim 64 or 128; "gte-encoder-neuron-kernels": right-padding mask).
//
// How (B200 design, not the pages' SBUF/PSUM one):
//   * one CTA owns 2 query tiles of 128 rows of one (b, h) and streams the
//     whole key sequence in 128-key tiles through a TMA ring in shared memory;
//   * warp 9 (one elected thread) issues tcgen05.mma: S_t = Q_t K^T into a
//     TMEM fp32 accumulator per query tile, then O_t += P_t V with P_t read
//     back from TMEM (bf16, aliased over S_t) and O_t an fp32 TMEM accumulator;
//   * warps 0-3 / 4-7 are the softmax warpgroups of query tiles 0 / 1: each
//     thread owns one query row (one TMEM lane), keeps the running max m and
//     sum l in fp32 registers, writes P, and rescales its O row in TMEM only
//     when the row max grew by more than 2^8 (the final O / l uses the same m,
//     so a stale m is exact);
//   * warp 8 (one elected thread) is the TMA producer.
// The two query tiles ping-pong: while one warpgroup computes exponentials the
// tensor core runs the other tile's MMAs.
#pragma once

#include "ptx.cuh"

namespace attn {
namespace enc {

constexpr int kTileM = 128;            // query rows per tile = TMEM lanes
constexpr int kTileN = 128;            // keys per K/V tile
constexpr int kQTiles = 2;             // query tiles per CTA
constexpr int kRowsPerCta = kTileM * kQTiles;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;          // 8 softmax warps + producer + MMA
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
    static constexpr int kPanels = D / 64;              // 128-byte swizzle panels per row
    static constexpr int kPanelBytes = 128 * 128;       // 128 rows x 128 bytes
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQTiles * kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_ready[2], o_final
    static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + tmem slot, abort flag, alignment slack
    // TMEM columns
    static constexpr uint32_t kColS0 = 0;
    static constexpr uint32_t kColO0 = 256;
};

struct Bars {
    uint64_t* q_full;
    uint64_t* k_full;
    uint64_t* k_empty;
    uint64_t* v_full;
    uint64_t* v_empty;
    uint64_t* s_full;
    uint64_t* p_ready;
    uint64_t* o_final;
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
    using C = Cfg<D>;
    uint64_t* b = reinterpret_cast<uint64_t*>(base + C::kBarOff);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + C::kStages;
    r.v_full = r.k_empty + C::kStages;
    r.v_empty = r.v_full + C::kStages;
    r.s_full = r.v_empty + C::kStages;
    r.p_ready = r.s_full + 2;
    r.o_final = r.p_ready + 2;
    return r;
}

template <int D, bool kHasBias>
__global__ void __launch_bounds__(kThreads, 1)
encoder_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out,
                   const float* __restrict__ key_bias, int H, int S, float scale_log2) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Bars bars = carve_bars<D>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int bh = blockIdx.y;
    const int row0 = blockIdx.x * kRowsPerCta;
    const int n_kv = (S + kTileN - 1) / kTileN;

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars.s_full[t], 1);
            mbar_init(&bars.p_ready[t], kTileM);
        }
        mbar_init(bars.o_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane_id() == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane_id() == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(bars.q_full, kQTiles * C::kTileBytes);
            for (int t = 0; t < kQTiles; ++t)
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kQOff + t * C::kTileBytes + p * C::kPanelBytes, &tm_q,
                                bars.q_full, p * 64, row0 + t * kTileM, bh);
            int issued = 0;
            for (int j = 0; j < n_kv && ok; ++j) {
                const int st = j % C::kStages;
                const uint32_t use = j / C::kStages;
                if (use > 0) ok = mbar_wait(&bars.k_empty[st], (use - 1) & 1, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars.k_full[st], C::kTileBytes);
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kKOff + st * C::kTileBytes + p * C::kPanelBytes, &tm_k,
                                &bars.k_full[st], p * 64, j * kTileN, bh);
                if (use > 0) ok = mbar_wait(&bars.v_empty[st], (use - 1) & 1, abort_flag);
                if (!ok) { issued = j + 1; break; }
                mbar_arrive_expect_tx(&bars.v_full[st], C::kTileBytes);
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kVOff + st * C::kTileBytes + p * C::kPanelBytes, &tm_v,
                                &bars.v_full[st], p * 64, j * kTileN, bh);
                issued = j + 1;
            }
            if (!ok) {
                // let every copy this thread started land before the CTA exits
                mbar_wait_drain(bars.q_full, 0);
                for (int j = (issued > C::kStages ? issued - C::kStages : 0); j < issued; ++j) {
                    const int st = j % C::kStages;
                    mbar_wait_drain(&bars.k_full[st], (j / C::kStages) & 1);
                    mbar_wait_drain(&bars.v_full[st], (j / C::kStages) & 1);
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane_id() == 0) {
            constexpr uint32_t idesc_qk = make_idesc(kTileM, kTileN, 1, 1, 0, 0);
            constexpr uint32_t idesc_pv = make_idesc(kTileM, D, 1, 1, 0, 1);
            const uint32_t q_addr = smem_u32(smem + C::kQOff);
            const uint32_t k_addr = smem_u32(smem + C::kKOff);
            const uint32_t v_addr = smem_u32(smem + C::kVOff);
            bool ok = mbar_wait(bars.q_full, 0, abort_flag);

            // S_t = Q_t K_j^T : K-steps of 16 along D (32 bytes inside a 128-byte panel row)
            auto issue_qk = [&](int t, int st) {
                const uint32_t qa = q_addr + t * C::kTileBytes;
                const uint32_t ka = k_addr + st * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk / 4) * C::kPanelBytes + (kk % 4) * 32;
                    mma_f16_ss(tmem_base + C::kColS0 + t * 128, smem_desc(qa + off, 16, 1024),
                               smem_desc(ka + off, 16, 1024), idesc_qk, kk > 0);
                }
            };
            // O_t += P_t V_j : A = P_t in TMEM (bf16 pairs over S_t columns), B = V (MN-major)
            auto issue_pv = [&](int t, int st, bool acc) {
                const uint32_t va = v_addr + st * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk) {
                    mma_f16_ts(tmem_base + C::kColO0 + t * D, tmem_base + C::kColS0 + t * 128 + kk * 8,
                               smem_desc(va + kk * 16 * 128, C::kPanelBytes, 1024), idesc_pv,
                               (acc || kk > 0) ? 1u : 0u);
                }
            };

            if (ok) ok = mbar_wait(&bars.k_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_qk(0, 0);
                tc_commit(&bars.s_full[0]);
                issue_qk(1, 0);
                tc_commit(&bars.s_full[1]);
                tc_commit(&bars.k_empty[0]);
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                const int st = j % C::kStages;
                const uint32_t ph = (j / C::kStages) & 1;
                const int stn = (j + 1) % C::kStages;
                const uint32_t phn = ((j + 1) / C::kStages) & 1;
                const bool more = (j + 1) < n_kv;
                ok = mbar_wait(&bars.v_full[st], ph, abort_flag);
                if (ok) ok = mbar_wait(&bars.p_ready[0], j & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_pv(0, st, j > 0);
                if (more) {
                    ok = mbar_wait(&bars.k_full[stn], phn, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(0, stn);
                    tc_commit(&bars.s_full[0]);
                }
                ok = mbar_wait(&bars.p_ready[1], j & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_pv(1, st, j > 0);
                if (more) {
                    issue_qk(1, stn);
                    tc_commit(&bars.s_full[1]);
                    tc_commit(&bars.k_empty[stn]);
                }
                tc_commit(&bars.v_empty[st]);
            }
            // o_final fires when every MMA above has completed (also on the abort path,
            // so that TMEM is quiescent before it is freed)
            tc_commit(bars.o_final);
            if (!ok) mbar_wait_drain(bars.o_final, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp >> 2;                        // query tile of this warpgroup
        const int r = threadIdx.x & 127;                // row inside the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem_base + lane_off + C::kColS0 + t * 128;
        const uint32_t tO = tmem_base + lane_off + C::kColO0 + t * D;
        const int b = bh / H;
        float m_run = -INFINITY;   // running max, log2 units (scale folded in)
        float l_run = 0.f;
        bool ok = true;

        for (int j = 0; j < n_kv; ++j) {
            ok = mbar_wait(&bars.s_full[t], j & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            float s[kTileN];
            {
                uint32_t u[kTileN];
                tmem_ld128_wait(tS, u);
#pragma unroll
                for (int i = 0; i < kTileN; ++i) s[i] = __uint_as_float(u[i]);
            }
            const int kv0 = j * kTileN;
            const int valid = S - kv0;   // keys of this tile that exist
            float m_tile;
            if constexpr (kHasBias) {
                const float* kb = key_bias + static_cast<size_t>(b) * S + kv0;
#pragma unroll
                for (int i = 0; i < kTileN; ++i) {
                    const float bias = (i < valid) ? __ldg(kb + i) : -INFINITY;
                    s[i] = (bias == -INFINITY) ? -INFINITY : fmaf(s[i], scale_log2, bias * kLog2e);
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < kTileN; i += 4) {
                    mx[0] = fmaxf(mx[0], s[i]);
                    mx[1] = fmaxf(mx[1], s[i + 1]);
                    mx[2] = fmaxf(mx[2], s[i + 2]);
                    mx[3] = fmaxf(mx[3], s[i + 3]);
                }
                m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            } else {
                if (valid < kTileN) {
#pragma unroll
                    for (int i = 0; i < kTileN; ++i)
                        if (i >= valid) s[i] = -INFINITY;
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < kTileN; i += 4) {
                    mx[0] = fmaxf(mx[0], s[i]);
                    mx[1] = fmaxf(mx[1], s[i + 1]);
                    mx[2] = fmaxf(mx[2], s[i + 2]);
                    mx[3] = fmaxf(mx[3], s[i + 3]);
                }
                m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
            }
            const bool upd = m_tile > m_run + kRescaleThreshold;
            const float m_next = upd ? m_tile : m_run;
            const float m_use = (m_next == -INFINITY) ? 0.f : m_next;
            const float alpha = upd ? ex2_approx(m_run - m_use) : 1.f;
            // P = exp2(s * scale_log2 - m), row sum in fp32
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kTileN; ++i) {
                float p;
                if constexpr (kHasBias) p = ex2_approx(s[i] - m_use);
                else p = ex2_approx(fmaf(s[i], scale_log2, -m_use));
                s[i] = p;
                ls[i & 3] += p;
            }
            l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            m_run = m_next;
            // rescale this row of O (only if some row of the warp moved its max)
            if (j > 0 && __any_sync(0xffffffffu, upd)) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32_wait(tO + c * 32, u);
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
                    tmem_st32(tO + c * 32, u);
                }
            }
            // P (bf16 pairs) over the first 64 columns of S_t
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) u[i] = pack_bf16x2(s[c * 64 + 2 * i], s[c * 64 + 2 * i + 1]);
                tmem_st32(tS + c * 32, u);
            }
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_ready[t]);
        }
        if (ok) ok = mbar_wait(bars.o_final, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const int row = row0 + t * kTileM + r;
            const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
            uint16_t* orow = out + (static_cast<size_t>(bh) * S + row) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t u[32];
                tmem_ld32_wait(tO + c * 32, u);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
                if (row < S) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace enc
}  // namespace attn
