// encoder.cuh -- non-causal multi-head encoder attention forward at head_dim 128 (sm_100a).
//
// What it computes: out[b,h] = softmax(scale * Q K^T + key_bias[b]) V for
// q/k/v/out in [B, H, S, 128] bf16: the attention core of the ViT / NewBERT encoder pages
// ("V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2", "vit-encoder-neuron-kernels":
// bidirectional self-attention with head_dim 64 or 128; "gte-encoder-neuron-kernels":
// right-padding mask). Head dim 64 runs the one-query-tile kernel (encoder1q.cuh).
//
// How (B200 design, not the pages' SBUF/PSUM one):
//   * one CTA owns 2 query tiles of 128 rows of one (b, h) and streams the
//     whole key sequence in 128-key tiles through a TMA ring in shared memory;
//   * warp 17 (one elected thread) issues tcgen05.mma: S_t = Q_t K^T into a
//     TMEM fp32 accumulator per query tile, then O_t += P_t V with P_t read
//     back from TMEM (bf16, written over S_t: S and O of both tiles fill TMEM)
//     and O_t an fp32 TMEM accumulator;
//   * warps 0-7 / 8-15 are the softmax warpgroups of query tiles 0 / 1: a row
//     (one TMEM lane) is shared by two warps on the same scheduler, 64 S
//     columns each, which exchange their halves' maxima and sums through
//     shared memory; each keeps the running max m and sum l in fp32 registers,
//     writes P, and rescales its half of the O row in TMEM only when the row
//     max grew by more than 2^8 (the final O / l uses the same m, so a stale m
//     is exact); one column pair in eight takes 2^x from an FMA-pipe polynomial
//     instead of the MUFU unit;
//   * warp 16 (one elected thread) is the TMA producer; with a key bias the whole warp
//     also counts the key tiles up to the batch entry's last kept key (the tiles after it
//     are neither loaded nor computed) and stages each live tile's bias in log2 units in a
//     shared-memory ring, with a word that says whether the tile is a prefix mask (0 on
//     its first columns, -inf on the rest): such a tile runs the unbiased path with the
//     -inf part masked, any other adds the staged bias to its scores (one FMA per score),
//     and a dropped key weighs exactly 0 (its V row may hold any finite value).
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
// Warps 0-15 run the softmax: warp w serves query tile w / 8, half (w / 4) % 2 of the
// 128 S columns, TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31. Two warps share every row, so
// each scheduler holds four softmax warps to hide TMEM / MUFU / barrier latency.
constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 576;
// Of every 8 column pairs of an S tile on the unbiased path, this many take 2^x from the
// FMA-pipe polynomial instead of the MUFU ex2 unit (one in eight measured 1% faster than none).
constexpr int kPolyEighths = 1;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
    static_assert(D == 128, "head dim 64 runs the one-query-tile kernel");
    static constexpr int kPanels = D / 64;              // 128-byte swizzle panels per row
    static constexpr int kPanelBytes = 128 * 128;       // 128 rows x 128 bytes
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kStages = 2;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQTiles * kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_ready[2],
    // o_final, xchg[2] (row-max / row-sum exchange between the two halves of a tile),
    // count_ready (the number of key tiles with a kept key is known; key-bias kernels),
    // bias_full[S] / bias_empty[S] (a key tile's bias staged by the producer / read by every
    // softmax warp; key-bias kernels)
    static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1 + 2 + 1 + 2 * kStages;
    static constexpr int kXchgOff = kBarOff + kNumBars * 8;   // float [2 buf][2 tile][2 half][128]
    static constexpr int kMiscOff = kXchgOff + 2 * 2 * 2 * 128 * 4;   // tmem slot, abort flag, count
    // key-bias kernels: per ring stage the tile's bias in log2 units (128 floats) and one word,
    // the first -inf column when the tile is a prefix mask (zeros, then -inf), else -1
    static constexpr int kBiasOff = (kMiscOff + 16 + 15) & ~15;   // 16-byte stores
    static constexpr int kBiasInfoOff = kBiasOff + kStages * kTileN * 4;
    static constexpr int kSmemBytes = kBiasInfoOff + kStages * 4 + 1024;   // + alignment slack
    // TMEM columns: S_t at 128 t, O_t at 256 + D t. TMEM is full, so P_t (bf16 pairs) is
    // written over the first 64 columns of S_t.
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
    uint64_t* xchg;
    uint64_t* count_ready;
    uint64_t* bias_full;
    uint64_t* bias_empty;
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
    r.xchg = r.o_final + 1;
    r.count_ready = r.xchg + 2;
    r.bias_full = r.count_ready + 1;
    r.bias_empty = r.bias_full + C::kStages;
    return r;
}

// Key tiles up to the last key whose bias is not -inf (at least one), found by a whole warp:
// with right padding the trailing tiles hold only -inf keys, which take no part in any row.
__device__ __forceinline__ int live_key_tiles(const float* kb, int S) {
    int last = -1;
    for (int c = static_cast<int>(lane_id()); c < S; c += 32)
        if (__ldg(kb + c) != -INFINITY) last = c;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    return max(1, (last + kTileN) / kTileN);
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
    const int n_kv_all = (S + kTileN - 1) / kTileN;
    // with a key bias: the key tiles that hold a kept key (the producer counts them while the
    // first copies are in flight and publishes the count here)
    volatile int* n_live_slot = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);
    float* bias_s = reinterpret_cast<float*>(smem + C::kBiasOff);
    volatile int* bias_info = reinterpret_cast<volatile int*>(smem + C::kBiasInfoOff);

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
            mbar_init(&bars.p_ready[t], kSoftmaxWarps / 2);   // one arrival per softmax warp of the tile
            mbar_init(&bars.xchg[t], kSoftmaxWarps / 2);
        }
        mbar_init(bars.o_final, 1);
        mbar_init(bars.count_ready, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars.bias_full[s], 1);
            mbar_init(&bars.bias_empty[s], kSoftmaxWarps);   // every softmax warp reads it
        }
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
    // set-up done: let the next kernel on the stream start, then wait for the previous one
    pdl_launch_dependents();
    pdl_wait_predecessor();
    int issued_k = 0, issued_v = 0;   // producer: K / V tiles whose copies were started

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        bool ok = true;
        auto load_kv = [&](int j) {   // K and V tile j into ring stage j % kStages (lane 0)
            const int st = j % C::kStages;
            const uint32_t use = j / C::kStages;
            if (use > 0) ok = mbar_wait(&bars.k_empty[st], (use - 1) & 1, abort_flag);
            if (!ok) return;
            mbar_arrive_expect_tx(&bars.k_full[st], C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kKOff + st * C::kTileBytes + p * C::kPanelBytes, &tm_k,
                            &bars.k_full[st], p * 64, j * kTileN, bh);
            issued_k = j + 1;
            if (use > 0) ok = mbar_wait(&bars.v_empty[st], (use - 1) & 1, abort_flag);
            if (!ok) return;
            mbar_arrive_expect_tx(&bars.v_full[st], C::kTileBytes);
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(smem + C::kVOff + st * C::kTileBytes + p * C::kPanelBytes, &tm_v,
                            &bars.v_full[st], p * 64, j * kTileN, bh);
            issued_v = j + 1;
        };
        if (lane_id() == 0) {
            mbar_arrive_expect_tx(bars.q_full, kQTiles * C::kTileBytes);
            for (int t = 0; t < kQTiles; ++t)
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(smem + C::kQOff + t * C::kTileBytes + p * C::kPanelBytes, &tm_q,
                                bars.q_full, p * 64, row0 + t * kTileM, bh);
            load_kv(0);
        }
        __syncwarp();
        if constexpr (kHasBias) {
            const float* kb_row = key_bias + static_cast<size_t>(bh / H) * S;
            const int n_kv = live_key_tiles(kb_row, S);
            if (lane_id() == 0) {
                *n_live_slot = n_kv;
                mbar_arrive(bars.count_ready);   // release: the count is visible to the waiters
            }
            // Tile j's bias into ring stage j % kStages, whole warp, four columns per lane:
            // in log2 units (-inf kept, a finite value clamped at -FLT_MAX so that its key
            // stays), and whether the tile is a prefix mask: zeros up to its first -inf
            // column, -inf from there on (no bias, or the end of a right-padded entry).
            auto stage_bias = [&](int j) -> bool {
                const int st = j % C::kStages;
                const uint32_t use = j / C::kStages;
                if (use > 0 && !mbar_wait_warp(&bars.bias_empty[st], (use - 1) & 1, abort_flag)) return false;
                const int c = 4 * static_cast<int>(lane_id());
                const int valid = S - j * kTileN;
                float bv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) bv[e] = (c + e < valid) ? __ldg(kb_row + j * kTileN + c + e) : -INFINITY;
                int first_drop = kTileN;
#pragma unroll
                for (int e = 3; e >= 0; --e)
                    if (bv[e] == -INFINITY) first_drop = c + e;
                const int p = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<uint32_t>(first_drop)));
                bool prefix = true;
#pragma unroll
                for (int e = 0; e < 4; ++e) prefix = prefix && ((c + e < p) ? bv[e] == 0.f : bv[e] == -INFINITY);
                prefix = __all_sync(0xffffffffu, prefix);
                float w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) w[e] = bv[e] == -INFINITY ? -INFINITY : fmaxf(bv[e] * kLog2e, -FLT_MAX);
                reinterpret_cast<float4*>(bias_s + st * kTileN)[lane_id()] = make_float4(w[0], w[1], w[2], w[3]);
                if (lane_id() == 0) bias_info[st] = prefix ? p : -1;
                __syncwarp();
                if (lane_id() == 0) mbar_arrive(&bars.bias_full[st]);   // release: the stage is visible
                return true;
            };
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) ok = stage_bias(0);
            for (int j = 1; j < n_kv && ok; ++j) {
                if (lane_id() == 0) load_kv(j);
                ok = __shfl_sync(0xffffffffu, ok, 0);   // lane 0's copies decide for the warp
                if (ok) ok = stage_bias(j);
            }
        } else if (lane_id() == 0) {
            for (int j = 1; j < n_kv_all && ok; ++j) load_kv(j);
            // on an abort (here or in another role) the copies are drained at teardown
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

            // Descriptors are built once; a K-step or a ring stage only moves the start
            // address, i.e. adds (bytes >> 4) to the low word.
            const uint64_t dq = smem_desc(q_addr, 16, 1024);
            const uint64_t dk = smem_desc(k_addr, 16, 1024);
            const uint64_t dv = smem_desc(v_addr, C::kPanelBytes, 1024);
            // S_t = Q_t K_j^T : K-steps of 16 along D (32 bytes inside a 128-byte panel row)
            auto issue_qk = [&](int t, int st) {
                const uint64_t qa = dq + static_cast<uint64_t>((t * C::kTileBytes) >> 4);
                const uint64_t ka = dk + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
                const uint32_t d = tmem_base + C::kColS0 + t * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kPanelBytes + (kk % 4) * 32) >> 4);
                    mma_f16_ss(d, qa + off, ka + off, idesc_qk, kk > 0);
                }
            };
            // O_t += P_t V_j : A = P_t in TMEM (bf16 pairs over S_t columns), B = V (MN-major)
            auto issue_pv = [&](int t, int st, bool acc) {
                const uint64_t va = dv + static_cast<uint64_t>((st * C::kTileBytes) >> 4);
                const uint32_t d = tmem_base + C::kColO0 + t * D;
                const uint32_t a = tmem_base + C::kColS0 + t * 128;   // P_t over S_t
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    mma_f16_ts(d, a + kk * 8, va + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                               (acc || kk > 0) ? 1u : 0u);
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
            int n_kv = n_kv_all;
            if constexpr (kHasBias) {
                if (ok) ok = mbar_wait(bars.count_ready, 0, abort_flag);
                n_kv = *n_live_slot;
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
            // o_final fires when every MMA above has completed (committed on the abort path
            // too: teardown waits for it before TMEM is freed)
            tc_commit(bars.o_final);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        constexpr int kHalf = kTileN / 2;                // S columns per warp
        const int t = warp >> 3;                         // query tile
        const int hf = (warp >> 2) & 1;                  // which half of the S columns
        const int r = ((warp & 3) << 5) | static_cast<int>(lane_id());   // row in the tile
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem_base + lane_off + C::kColS0 + t * 128;
        const uint32_t tSh = tS + hf * kHalf;            // this warp's S columns
        const uint32_t tPh = tS + hf * (kHalf / 2);    // this warp's P columns (over S)
        const uint32_t tOh = tmem_base + lane_off + C::kColO0 + t * D + hf * (D / 2);
        float* xchg = reinterpret_cast<float*>(smem + C::kXchgOff);
        auto xslot = [&](int buf, int half) { return xchg + ((buf * 2 + t) * 2 + half) * kTileM + r; };
        const int col0 = hf * kHalf;
        float m_run = -INFINITY;   // running max, log2 units (scale folded in)
        float l_run = 0.f;         // running sum over this warp's half of the columns
        bool ok = true;
        int n_kv = n_kv_all;
        if constexpr (kHasBias) {
            ok = mbar_wait_warp(bars.count_ready, 0, abort_flag);
            n_kv = *n_live_slot;
        }
        // publish v in slot `buf` and read the partner half's value once both are in
        auto exchange = [&](float v, int buf, uint32_t phase, float* other) -> bool {
            *xslot(buf, hf) = v;
            __threadfence_block();
            tc_fence_before();   // this warp's TMEM reads of S precede the partner's P writes
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&bars.xchg[t]);
            if (!mbar_wait_warp(&bars.xchg[t], phase, abort_flag)) return false;
            tc_fence_after();
            *other = *xslot(buf, hf ^ 1);
            return true;
        };

        for (int j = 0; ok && j < n_kv; ++j) {
            ok = mbar_wait_warp(&bars.s_full[t], j & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const int kv0 = j * kTileN;
            int valid = S - kv0;   // keys of this tile that take part (the rest are -inf)
            bool raw_path = true;
            const float* bl = nullptr;
            if constexpr (kHasBias) {
                // the producer has staged this tile's bias: a prefix mask (zeros, then -inf: no
                // bias, or the end of a right-padded entry) is computed as without a bias with
                // its -inf part masked like the columns past S; any other tile adds the staged
                // log2-unit bias to its scores
                const int stb = j % C::kStages;
                ok = mbar_wait_warp(&bars.bias_full[stb], (j / C::kStages) & 1, abort_flag);
                if (!ok) break;
                const int info = bias_info[stb];
                raw_path = info >= 0;
                if (raw_path) {
                    valid = info;
                    __syncwarp();
                    if (lane_id() == 0) mbar_arrive(&bars.bias_empty[stb]);
                } else {
                    bl = bias_s + stb * kTileN + col0;
                }
            }
            uint32_t u[kHalf];
            tmem_ld64_wait(tSh, u);
            // On the raw-score path the columns past S (or past a prefix mask's end) become
            // -inf (the scale is positive, so the max is unchanged); their weights are 0, or
            // 2^-125 where the polynomial takes them against V rows that the copy zero-filled
            // (the key-bias build makes those weights exactly 0: a dropped key's V row may hold
            // any finite value).
            if (raw_path && valid < kTileN) {
#pragma unroll
                for (int i = 0; i < kHalf; ++i)
                    if (col0 + i >= valid) u[i] = __float_as_uint(-INFINITY);
            }
            float m_half;
            if (raw_path) {
                // pairs first, then three-input maxes over groups of 8 columns
                static_assert(kHalf % 8 == 0, "row max reads whole groups of 8 columns");
                float mx[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    mx[e] = fmaxf(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
#pragma unroll
                for (int i = 8; i < kHalf; i += 8) {
                    mx[0] = fmax3(mx[0], __uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                    mx[1] = fmax3(mx[1], __uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
                    mx[2] = fmax3(mx[2], __uint_as_float(u[i + 4]), __uint_as_float(u[i + 5]));
                    mx[3] = fmax3(mx[3], __uint_as_float(u[i + 6]), __uint_as_float(u[i + 7]));
                }
                m_half = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * scale_log2;
            } else if constexpr (kHasBias) {
                // biased score in log2 units: one packed FMA per two scores against the staged
                // bias (-inf where the key is dropped or past S: the staged value is -inf there)
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < kHalf; i += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(bl + i);
                    const float2 x01 = __ffma2_rn(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                                  make_float2(scale_log2, scale_log2), make_float2(b4.x, b4.y));
                    const float2 x23 = __ffma2_rn(make_float2(__uint_as_float(u[i + 2]), __uint_as_float(u[i + 3])),
                                                  make_float2(scale_log2, scale_log2), make_float2(b4.z, b4.w));
                    u[i] = __float_as_uint(x01.x);
                    u[i + 1] = __float_as_uint(x01.y);
                    u[i + 2] = __float_as_uint(x23.x);
                    u[i + 3] = __float_as_uint(x23.y);
                    mx[0] = fmaxf(mx[0], x01.x);
                    mx[1] = fmaxf(mx[1], x01.y);
                    mx[2] = fmaxf(mx[2], x23.x);
                    mx[3] = fmaxf(mx[3], x23.y);
                }
                __syncwarp();
                if (lane_id() == 0) mbar_arrive(&bars.bias_empty[j % C::kStages]);
                m_half = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            }
            float m_other;
            ok = exchange(m_half, j & 1, j & 1, &m_other);
            if (!ok) break;
            const float m_tile = fmaxf(m_half, m_other);
            const bool upd = m_tile > m_run + kRescaleThreshold;
            const float m_next = upd ? m_tile : m_run;
            const float m_use = (m_next == -INFINITY) ? 0.f : m_next;
            const float alpha = upd ? ex2_approx(m_run - m_use) : 1.f;
            // P = 2^(score - m) as bf16 pairs, 16 words at a time; row sum in fp32
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kHalf / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int kk = c * 16 + k;   // column pair index in this half
                    const float2 sv = make_float2(__uint_as_float(u[2 * kk]), __uint_as_float(u[2 * kk + 1]));
                    float2 pv;
                    if (raw_path) {
                        const float2 x = __ffma2_rn(sv, make_float2(scale_log2, scale_log2),
                                                    make_float2(-m_use, -m_use));
                        if ((kk & 7) < kPolyEighths) {
                            pv = exp2_poly2(x);
                            if constexpr (kHasBias) {   // a dropped key weighs exactly 0
                                if (x.x == -INFINITY) pv.x = 0.f;
                                if (x.y == -INFINITY) pv.y = 0.f;
                            }
                        } else {
                            pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        }
                    } else {
                        pv = make_float2(ex2_approx(sv.x - m_use), ex2_approx(sv.y - m_use));
                    }
                    if (k & 1) acc1 = __fadd2_rn(acc1, pv);
                    else acc0 = __fadd2_rn(acc0, pv);
                    pk[k] = pack_bf16x2(pv.x, pv.y);
                }
                // P over S: s_full of this tile implied that PV_t of the previous one is done.
                // Both halves read their S columns before the exchange above, so P columns
                // that overlap the first half's S columns are free to write.
                tmem_st16(tPh + c * 16, pk);
            }
            if (!ok) break;
            l_run = l_run * alpha + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
            m_run = m_next;
            // rescale this warp's half of the O row (only if some row of the warp moved its max)
            if (j > 0 && __any_sync(0xffffffffu, upd)) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t w[32];
                    tmem_ld32_wait(tOh + c * 32, w);
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
                    tmem_st32(tOh + c * 32, w);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&bars.p_ready[t]);
        }
        // full row sum = both halves
        float l_other = 0.f;
        if (ok) ok = exchange(l_run, n_kv & 1, n_kv & 1, &l_other);
        if (ok) ok = mbar_wait_warp(bars.o_final, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const float l_tot = l_run + l_other;
            const int row = row0 + t * kTileM + r;
            const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
            uint16_t* orow = out + (static_cast<size_t>(bh) * S + row) * D + hf * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t w[32];
                tmem_ld32_wait(tOh + c * 32, w);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(w[2 * i]) * inv_l, __uint_as_float(w[2 * i + 1]) * inv_l);
                if (row < S) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
        tc_wait_st();   // no TMEM store of this warp is in flight when TMEM is freed
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // Some role gave up (a bounded wait ran out): nothing of this CTA may still be in
        // flight when it exits. Every copy the producer started lands in shared memory (the
        // latest fill of each ring stage; earlier fills were consumed before their stage was
        // refilled), and every MMA completes before TMEM is freed.
        if (warp == kProducerWarp && lane_id() == 0) {
            mbar_wait_drain(bars.q_full, 0);
            for (int j = (issued_k > C::kStages ? issued_k - C::kStages : 0); j < issued_k; ++j)
                mbar_wait_drain(&bars.k_full[j % C::kStages], (j / C::kStages) & 1);
            for (int j = (issued_v > C::kStages ? issued_v - C::kStages : 0); j < issued_v; ++j)
                mbar_wait_drain(&bars.v_full[j % C::kStages], (j / C::kStages) & 1);
        }
        if (warp == kMmaWarp && lane_id() == 0) mbar_wait_drain(bars.o_final, 0);
        __syncwarp();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace enc
}  // namespace attn
