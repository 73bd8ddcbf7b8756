// paged.cuh -- history-only attention over a paged FP8 (E4M3FN) KV cache, sm_100a.
//
// What it computes ("Prefill Context-Parallel Attention POC for Trainium2",
// sections "Layout", the history-only rule, the additive bias from
// actual_history_len, "Current POC constraints"): for query head h, query row
// i and kv head g = h / num_kv_groups,
//   out[h, i] = softmax_t(scale * q[h,i] . K_t) V_t  over t < actual_history_len,
// where logical position t is row t % block_size of physical block
// block_table[t / block_size] and K_t = k_scale * code, V_t = v_scale * code.
//
// How (B200 design):
//   * one CTA owns 128 query rows of one head; the loop runs over 128-key
//     sub-tiles of the logical history (a 512-token block is 4 sub-tiles) -- the
//     page's ring of ranks becomes this loop over the blocks the table names;
//     sub-tiles at or past actual_history_len are never loaded;
//   * the producer warp reads block_table and TMA-loads the FP8 K and V tiles
//     straight from the pool (no gather copy, no dequantisation pass);
//   * both matmuls run as FP8 tcgen05 MMAs (kind::f8f6f4) on the stored codes.
//     The tensor cores cannot mix bf16 with fp8, so the bf16 operand of each
//     matmul is split into two e4m3 terms, x ~ hi + lo (lo = e4m3(x - hi)):
//       S = (Q_hi + Q_lo) K^T  -- Q quantised once per CTA with a per-row scale,
//       O += (P_hi + P_lo) V   -- P scaled by 2^7 so it sits in e4m3's normal range.
//     Each split costs a second MMA into the same fp32 TMEM accumulator and keeps
//     the result at bf16-level accuracy (a single e4m3 term would not);
//   * S is double-buffered in TMEM so QK of the next sub-tile runs while the
//     softmax warpgroup works; P_hi / P_lo are written back over S and read by
//     the MMA from TMEM; O (128 x 256 fp32) stays in TMEM for the whole loop.
//
// Prefill with current tokens (the same kernel, `Params::seq_q_start` set): the page's
// "current tokens do not attend to one another yet", completed. Several sequences per
// launch (blockIdx.z); sequence s owns q rows seq_q_start[s] .. seq_q_start[s+1] - 1,
// its block-table row and history length seq_hist[s]; its current tokens' K/V are in
// the cache after the history. Query i (logical position hist + i) sees every position
// t <= hist + i: each softmax row masks its own limit, and a CTA loads only the
// sub-tiles its last row can see.
#pragma once

#include "ptx.cuh"
#include "tmap.cuh"

namespace attn {
namespace paged {

constexpr int kD = 256;
constexpr int kTileM = 128;
constexpr int kTileN = 128;                 // keys per sub-tile
constexpr int kThreads = 192;               // softmax warpgroup + producer + MMA
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0;              // S buffers at 0 and 128
constexpr uint32_t kColO = 256;             // O: 256 fp32 columns
constexpr float kRescaleThreshold = 1.0f;   // log2 units: p <= 2 before the 2^7 scale
constexpr float kPScaleLog2 = 7.0f;         // P is stored as p * 2^7 (<= 256 < 448)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStages = 2;

constexpr int kPanel = 128 * 128;                     // 128 rows x 128 bytes
constexpr int kQ8Bytes = 2 * kPanel;                  // 128 rows x 256 fp8
constexpr int kKVTileBytes = 2 * kPanel;              // 128 keys x 256 fp8
constexpr int kQhOff = 0;
constexpr int kQlOff = kQhOff + kQ8Bytes;
constexpr int kKOff = kQlOff + kQ8Bytes;
constexpr int kVOff = kKOff + kStages * kKVTileBytes;
constexpr int kStageOff = kKOff;                      // bf16 Q staging (64 KB) aliases the ring
constexpr int kBarOff = kVOff + kStages * kKVTileBytes;
constexpr int kNumBars = 1 + 1 + 4 * kStages + 2 + 1 + 1 + 1;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kSmemBytes = kMiscOff + 16 + 1024;
static_assert(kStages * 2 * kKVTileBytes >= 4 * kPanel, "staging must fit in the ring");

struct Bars {
    uint64_t *q_full, *q_ready, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_ready, *o_ready,
        *o_final;
};

__device__ __forceinline__ Bars carve(uint8_t* smem) {
    uint64_t* b = reinterpret_cast<uint64_t*>(smem + kBarOff);
    Bars r;
    r.q_full = b;
    r.q_ready = b + 1;
    r.k_full = b + 2;
    r.k_empty = r.k_full + kStages;
    r.v_full = r.k_empty + kStages;
    r.v_empty = r.v_full + kStages;
    r.s_full = r.v_empty + kStages;
    r.p_ready = r.s_full + 2;
    r.o_ready = r.p_ready + 1;
    r.o_final = r.o_ready + 1;
    return r;
}

struct Params {
    uint16_t* out;
    const int32_t* block_table;     // history mode: the table; prefill: row 0 of [num_seqs][table_stride]
    int Sq, Hkv, G, num_phys_blocks, block_size, hist_len;
    float c_qk;        // k_scale * softmax_scale * log2(e)   (times the per-row Q scale)
    float v_scale;
    // prefill with current tokens (nullptr: one sequence, history only)
    const int32_t* seq_q_start;     // [num_seqs + 1]
    const int32_t* seq_hist;        // [num_seqs]
    int table_stride;               // block-table entries per sequence
};

// Logical 128-key sub-tile j -> (physical block, row offset); -1 if the table entry is bad.
__device__ __forceinline__ int sub_tile_block(const Params& p, const int32_t* table, int j, int* off) {
    const int t0 = j * kTileN;
    const int lb = t0 / p.block_size;
    *off = t0 - lb * p.block_size;
    const int phys = __ldg(table + lb);
    return (phys >= 0 && phys < p.num_phys_blocks) ? phys : -1;
}

__global__ void __launch_bounds__(kThreads, 1)
paged_history_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Bars bars = carve(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int h = blockIdx.y;
    const int g = h / p.G;
    const int row0 = blockIdx.x * kTileM;   // first query row of the tile, within its sequence

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        mbar_init(bars.q_ready, kTileM);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.v_empty[s], 1);
        }
        mbar_init(&bars.s_full[0], 1);
        mbar_init(&bars.s_full[1], 1);
        mbar_init(bars.p_ready, kTileM);
        mbar_init(bars.o_ready, 1);
        mbar_init(bars.o_final, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait_predecessor();

    // this CTA's sequence: q rows [q0, q0 + q_len), history length, block-table row
    int q0 = 0, q_len = p.Sq, hist = p.hist_len;
    const int32_t* table = p.block_table;
    const bool causal = p.seq_q_start != nullptr;
    bool active = true;
    if (causal) {
        const int s = blockIdx.z;
        q0 = __ldg(p.seq_q_start + s);
        q_len = __ldg(p.seq_q_start + s + 1) - q0;
        hist = __ldg(p.seq_hist + s);
        table = p.block_table + static_cast<size_t>(s) * p.table_stride;
        if (q0 < 0 || q_len < 0 || q0 + q_len > p.Sq || hist < 0 ||
            static_cast<long long>(hist) + q_len > static_cast<long long>(p.table_stride) * p.block_size) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
                record_status(-9 /* ATTN_ERR_SEQUENCE */);
            active = false;
        }
    }
    active = active && row0 < q_len;
    // keys [0, key_end) are visible to some row of the tile
    const int key_end = causal ? hist + min(row0 + kTileM, q_len) : hist;
    const int n_sub = active ? (key_end + kTileN - 1) / kTileN : 0;
    bool q_issued = false;            // producer: the Q copy was started
    int issued_k = 0, issued_v = 0;   // producer: K / V sub-tiles whose copies were started

    if (!active) {
        // nothing to compute or store (rows past the sequence, or a bad descriptor)
    } else if (warp == kProducerWarp) {
        // ---------------------------------------------------------------- producer
        if (lane_id() == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            mbar_arrive_expect_tx(bars.q_full, 4 * kPanel);
            for (int pn = 0; pn < 4; ++pn)
                tma_load_3d(smem + kStageOff + pn * kPanel, &tm_q, bars.q_full, pn * 64, q0 + row0, h);
            q_issued = true;
            // the ring doubles as Q staging until the softmax warps have quantised Q
            bool ok = mbar_wait(bars.q_ready, 0, abort_flag);
            for (int j = 0; j < n_sub && ok; ++j) {
                const int st = j % kStages;
                const uint32_t use = j / kStages;
                int off;
                int phys = sub_tile_block(p, table, j, &off);
                if (phys < 0) {
                    record_status(-8 /* ATTN_ERR_BLOCK_TABLE */);
                    phys = 0;   // load something valid; the softmax masks the whole sub-tile
                }
                const int c2 = phys * p.Hkv + g;
                if (use > 0) ok = mbar_wait(&bars.k_empty[st], (use - 1) & 1, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars.k_full[st], kKVTileBytes);
                tma_load_3d(smem + kKOff + st * kKVTileBytes, &tm_k, &bars.k_full[st], 0, off, c2);
                tma_load_3d(smem + kKOff + st * kKVTileBytes + kPanel, &tm_k, &bars.k_full[st], 128,
                            off, c2);
                issued_k = j + 1;
                if (use > 0) ok = mbar_wait(&bars.v_empty[st], (use - 1) & 1, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars.v_full[st], kKVTileBytes);
                tma_load_3d(smem + kVOff + st * kKVTileBytes, &tm_v, &bars.v_full[st], 0, off, c2);
                tma_load_3d(smem + kVOff + st * kKVTileBytes + kPanel, &tm_v, &bars.v_full[st], 128,
                            off, c2);
                issued_v = j + 1;
            }
            // on an abort (here or in another role) the copies are drained at teardown
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane_id() == 0) {
            constexpr uint32_t idesc_qk = make_idesc(kTileM, kTileN, 0, 0, 0, 0);   // e4m3 x e4m3
            constexpr uint32_t idesc_pv = make_idesc(kTileM, kD, 0, 0, 0, 1);       // V MN-major
            const uint32_t qh = smem_u32(smem + kQhOff);
            const uint32_t ql = smem_u32(smem + kQlOff);
            const uint32_t ka = smem_u32(smem + kKOff);
            const uint32_t va = smem_u32(smem + kVOff);
            bool ok = mbar_wait(bars.q_ready, 0, abort_flag);
            // S_b = (Q_hi + Q_lo) K^T: 8 K-steps of 32 bytes per term
            auto issue_qk = [&](int b, int st) {
                const uint32_t kb = ka + st * kKVTileBytes;
                const uint32_t d = tmem_base + kColS0 + b * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk / 4) * kPanel + (kk % 4) * 32;
                    mma_f8_ss(d, smem_desc(qh + off, 16, 1024), smem_desc(kb + off, 16, 1024), idesc_qk,
                              kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk / 4) * kPanel + (kk % 4) * 32;
                    mma_f8_ss(d, smem_desc(ql + off, 16, 1024), smem_desc(kb + off, 16, 1024), idesc_qk, 1);
                }
            };
            // O += (P_hi + P_lo) V: A from TMEM (P_hi in S_b columns [0,32), P_lo in [32,64))
            auto issue_pv = [&](int b, int st, bool acc) {
                const uint32_t vb = va + st * kKVTileBytes;
                const uint32_t s = tmem_base + kColS0 + b * 128;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f8_ts(tmem_base + kColO, s + kk * 8, smem_desc(vb + kk * 32 * 128, kPanel, 1024),
                              idesc_pv, (acc || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f8_ts(tmem_base + kColO, s + 32 + kk * 8,
                              smem_desc(vb + kk * 32 * 128, kPanel, 1024), idesc_pv, 1u);
            };
            if (ok && n_sub > 0) {
                ok = mbar_wait(&bars.k_full[0], 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    issue_qk(0, 0);
                    tc_commit(&bars.s_full[0]);
                    tc_commit(&bars.k_empty[0]);
                }
            }
            for (int j = 0; j < n_sub && ok; ++j) {
                const int st = j % kStages;
                if (j + 1 < n_sub) {
                    const int stn = (j + 1) % kStages;
                    ok = mbar_wait(&bars.k_full[stn], ((j + 1) / kStages) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk((j + 1) & 1, stn);
                    tc_commit(&bars.s_full[(j + 1) & 1]);
                    tc_commit(&bars.k_empty[stn]);
                }
                ok = mbar_wait(bars.p_ready, j & 1, abort_flag);
                if (ok) ok = mbar_wait(&bars.v_full[st], (j / kStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_pv(j & 1, st, j > 0);
                tc_commit(bars.o_ready);
                tc_commit(&bars.v_empty[st]);
            }
            tc_commit(bars.o_final);   // teardown waits for it on an abort
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax warpgroup
        const int r = threadIdx.x;                       // 0..127: query row in the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        bool ok = mbar_wait_warp(bars.q_full, 0, abort_flag);
        float c_row = 0.f;
        if (ok) {
            // quantise this thread's Q row: x = sq * (hi + lo), sq = amax / 448 (per row)
            uint32_t w[128];
            const uint8_t* stage = smem + kStageOff;
#pragma unroll
            for (int pn = 0; pn < 4; ++pn)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v4 = *reinterpret_cast<const uint4*>(
                        stage + pn * kPanel + r * 128 + ((c ^ (r & 7)) << 4));
                    w[pn * 32 + c * 4 + 0] = v4.x;
                    w[pn * 32 + c * 4 + 1] = v4.y;
                    w[pn * 32 + c * 4 + 2] = v4.z;
                    w[pn * 32 + c * 4 + 3] = v4.w;
                }
            uint32_t amax_bits = 0;
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                amax_bits = max(amax_bits, (w[i] << 16) & 0x7FFFFFFFu);
                amax_bits = max(amax_bits, w[i] & 0x7FFF0000u);
            }
            const float amax = __uint_as_float(amax_bits);
            const float sq = amax > 0.f ? amax * (1.0f / 448.0f) : 1.0f;
            const float inv = 1.0f / sq;
            c_row = sq * p.c_qk;
            uint8_t* qh = smem + kQhOff;
            uint8_t* ql = smem + kQlOff;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {            // 16 chunks of 16 elements
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {        // 4 elements per 32-bit word
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t bw = w[ch * 8 + q4 * 2 + e];
                        x[2 * e] = __uint_as_float(bw << 16) * inv;
                        x[2 * e + 1] = __uint_as_float(bw & 0xFFFF0000u) * inv;
                    }
                    const uint32_t h01 = cvt_e4m3x2_f32(x[0], x[1]);
                    const uint32_t h23 = cvt_e4m3x2_f32(x[2], x[3]);
                    const float2 b01 = f16x2_to_f32x2(cvt_f16x2_e4m3x2(h01));
                    const float2 b23 = f16x2_to_f32x2(cvt_f16x2_e4m3x2(h23));
                    const uint32_t l01 = cvt_e4m3x2_f32(x[0] - b01.x, x[1] - b01.y);
                    const uint32_t l23 = cvt_e4m3x2_f32(x[2] - b23.x, x[3] - b23.y);
                    hw[q4] = h01 | (h23 << 16);
                    lw[q4] = l01 | (l23 << 16);
                }
                const int pn = ch / 8, c = ch % 8;
                const int so = pn * kPanel + r * 128 + ((c ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(qh + so) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(ql + so) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            fence_proxy_async_smem();   // generic-proxy writes -> visible to the MMA (async proxy)
        }
        mbar_arrive(bars.q_ready);      // also frees the staging area for K/V

        float m_run = -INFINITY;        // running max (log2 units)
        float l_run = 0.f;              // running sum of 2^7 * p
        const uint32_t tO = tmem_base + lane_off + kColO;
        for (int j = 0; j < n_sub && ok; ++j) {
            const int b = j & 1;
            const uint32_t tS = tmem_base + lane_off + kColS0 + b * 128;
            int off;
            const bool blk_ok = sub_tile_block(p, table, j, &off) >= 0;
            // this row sees keys [0, lim): the history, plus current tokens up to itself
            const int lim = causal ? hist + row0 + r + 1 : hist;
            const int valid = blk_ok ? max(0, min(kTileN, lim - j * kTileN)) : 0;
            ok = mbar_wait_warp(&bars.s_full[b], (j >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            float s[kTileN];
            {
                uint32_t u[kTileN];
                tmem_ld128_wait(tS, u);
#pragma unroll
                for (int i = 0; i < kTileN; ++i) s[i] = __uint_as_float(u[i]);
            }
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
            const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c_row;
            const bool upd = m_tile > m_run + kRescaleThreshold;
            const float m_next = upd ? m_tile : m_run;
            const float m_use = (m_next == -INFINITY) ? 0.f : m_next;
            const float alpha = upd ? ex2_approx(m_run - m_use) : 1.f;
            const float bias = kPScaleLog2 - m_use;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kTileN; ++i) {
                const float pv = ex2_approx(fmaf(s[i], c_row, bias));
                s[i] = pv;
                ls[i & 3] += pv;
            }
            l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            m_run = m_next;
            // P -> e4m3 hi / lo (via an exact f16 residual), four per TMEM column
            uint32_t ph[32], pl[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const uint32_t f01 = cvt_f16x2_f32(s[4 * c], s[4 * c + 1]);
                const uint32_t f23 = cvt_f16x2_f32(s[4 * c + 2], s[4 * c + 3]);
                const uint32_t h01 = cvt_e4m3x2_f16x2(f01);
                const uint32_t h23 = cvt_e4m3x2_f16x2(f23);
                const uint32_t l01 = cvt_e4m3x2_f16x2(hsub2(f01, cvt_f16x2_e4m3x2(h01)));
                const uint32_t l23 = cvt_e4m3x2_f16x2(hsub2(f23, cvt_f16x2_e4m3x2(h23)));
                ph[c] = h01 | (h23 << 16);
                pl[c] = l01 | (l23 << 16);
            }
            // O and the P buffer are free once PV of the previous sub-tile has completed
            if (j > 0) {
                ok = mbar_wait_warp(bars.o_ready, (j - 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, upd)) {
#pragma unroll
                    for (int c = 0; c < kD / 32; ++c) {
                        uint32_t u[32];
                        tmem_ld32_wait(tO + c * 32, u);
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
                        tmem_st32(tO + c * 32, u);
                    }
                }
            }
            tmem_st32(tS, ph);
            tmem_st32(tS + 32, pl);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(bars.p_ready);
        }
        if (ok) ok = mbar_wait_warp(bars.o_final, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const int row = row0 + r;
            uint16_t* orow = p.out + (static_cast<size_t>(h) * p.Sq + q0 + row) * kD;
            const bool live = l_run > 0.f;
            const float f = live ? p.v_scale / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t u[32];
                if (n_sub > 0) tmem_ld32_wait(tO + c * 32, u);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = live ? pack_bf16x2(__uint_as_float(u[2 * i]) * f, __uint_as_float(u[2 * i + 1]) * f)
                                 : 0u;
                if (row < q_len) {
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
        // Some role gave up (a bounded wait ran out): every copy the producer started lands
        // (the latest fill of each ring stage; earlier fills were consumed before their
        // stage was refilled) and every MMA completes before this CTA frees TMEM and exits.
        if (warp == kProducerWarp && lane_id() == 0) {
            if (q_issued) mbar_wait_drain(bars.q_full, 0);
            for (int j = (issued_k > kStages ? issued_k - kStages : 0); j < issued_k; ++j)
                mbar_wait_drain(&bars.k_full[j % kStages], (j / kStages) & 1);
            for (int j = (issued_v > kStages ? issued_v - kStages : 0); j < issued_v; ++j)
                mbar_wait_drain(&bars.v_full[j % kStages], (j / kStages) & 1);
        }
        if (warp == kMmaWarp && lane_id() == 0 && active) mbar_wait_drain(bars.o_final, 0);
        __syncwarp();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Shared set-up of both entry points: shared-memory opt-in, tensor maps, launch.
inline int launch_common(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                         int num_phys_blocks, int block_size, int Hq, int Hkv, int rows_q,
                         Params prm, dim3 grid, cudaStream_t stream) {
    static std::atomic<uint64_t> smem_done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -6;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(smem_done.load() & bit)) {
        if (cudaFuncSetAttribute(paged_history_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes) != cudaSuccess)
            return -6;
        smem_done.fetch_or(bit);
    }
    CUtensorMap tq, tk, tv;
    int rc;
    if ((rc = encode_map_3d_bf16(&tq, q, kD, rows_q, Hq, 64, kTileM))) return rc;
    const uint64_t planes = static_cast<uint64_t>(num_phys_blocks) * Hkv;
    if ((rc = encode_map_3d_u8(&tk, k_cache, kD, block_size, planes, 128, kTileN))) return rc;
    if ((rc = encode_map_3d_u8(&tv, v_cache, kD, block_size, planes, 128, kTileN))) return rc;
    return launch_pdl(paged_history_kernel, grid, dim3(kThreads), kSmemBytes, stream, tq, tk, tv, prm);
}

// History only: every query of one sequence sees logical positions [0, hist_len).
inline int launch(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                  const int32_t* block_table, int n_table, int num_phys_blocks, int block_size,
                  int hist_len, float k_scale, float v_scale, float softmax_scale, int Hq, int Hkv,
                  int G, int Sq, int D, uint16_t* out, cudaStream_t stream) {
    (void)n_table;
    (void)D;
    Params prm;
    prm.out = out;
    prm.block_table = block_table;
    prm.Sq = Sq;
    prm.Hkv = Hkv;
    prm.G = G;
    prm.num_phys_blocks = num_phys_blocks;
    prm.block_size = block_size;
    prm.hist_len = hist_len;
    prm.c_qk = k_scale * softmax_scale * kLog2e;
    prm.v_scale = v_scale;
    prm.seq_q_start = nullptr;
    prm.seq_hist = nullptr;
    prm.table_stride = 0;
    return launch_common(q, k_cache, v_cache, num_phys_blocks, block_size, Hq, Hkv, Sq, prm,
                         dim3((Sq + kTileM - 1) / kTileM, Hq), stream);
}

// Prefill: num_seqs sequences, each seeing its history and its current tokens causally.
inline int launch_prefill(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                          const int32_t* block_tables, int table_stride, int num_phys_blocks,
                          int block_size, const int32_t* q_start, const int32_t* hist_lens,
                          int num_seqs, int total_q, int max_q_len, float k_scale, float v_scale,
                          float softmax_scale, int Hq, int Hkv, int G, uint16_t* out,
                          cudaStream_t stream) {
    if (total_q == 0 || max_q_len == 0) return 0;
    Params prm;
    prm.out = out;
    prm.block_table = block_tables;
    prm.Sq = total_q;
    prm.Hkv = Hkv;
    prm.G = G;
    prm.num_phys_blocks = num_phys_blocks;
    prm.block_size = block_size;
    prm.hist_len = 0;
    prm.c_qk = k_scale * softmax_scale * kLog2e;
    prm.v_scale = v_scale;
    prm.seq_q_start = q_start;
    prm.seq_hist = hist_lens;
    prm.table_stride = table_stride;
    return launch_common(q, k_cache, v_cache, num_phys_blocks, block_size, Hq, Hkv, total_q, prm,
                         dim3((max_q_len + kTileM - 1) / kTileM, Hq, num_seqs), stream);
}

}  // namespace paged
}  // namespace attn
