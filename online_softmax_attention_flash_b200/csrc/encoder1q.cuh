// encoder1q.cuh -- non-causal encoder attention forward at head_dim 64, one query tile per
// CTA, two CTAs per SM (sm_100a).
//
// What it computes: the same as encoder_fwd_kernel (encoder.cuh), at D = 64: out[b,h] =
// softmax(scale * Q K^T + key_bias[b]) V, q/k/v/out [B, H, S, 64] bf16, key_bias [B, S] fp32
// additive or none. With a key bias (kHasBias) the producer warp counts the key tiles up to
// the entry's last kept key while the first copies fly (the tiles after it are never
// loaded), and stages each live tile's bias in log2 units in a shared-memory ring beside the
// K / V stages, with a word that says whether the tile is a prefix mask (0 on its first
// columns, -inf on the rest: no bias, or the end of a right-padded entry). A prefix-mask tile
// takes the unbiased path with the -inf part masked; any other tile adds the staged bias to
// its scores (one FMA per score) before the max. A dropped key (bias -inf) weighs exactly 0
// wherever the polynomial would give 2^-125, since its V row may hold any finite value.
//
// How. A CTA owns 128 query rows of one (b, h) and streams the key sequence in 128-key
// tiles through a 2-stage TMA ring: warp 5 (one thread) issues QK(j+1) as soon as the
// softmax has read S(j), and PV(j) in four 32-key parts, each as soon as the softmax warps
// have written that chunk of P(j) (one completion commit per tile: a commit per part costs
// more than the finer waits it would allow); warps 0-3 are the softmax, one thread per row
// holding all 128 scores of its row, so the row max needs no exchange between warps. TMEM
// holds S (128 columns), O (64) and P (64, bf16 pairs): 256 columns, and the CTA needs
// ~82 KB of shared memory, so two CTAs share an SM. The two query tiles
// an SM works on then belong to different CTAs: nothing in the issue order couples their
// phases, and one CTA's exponentials (MUFU) overlap the other's max, stores and waits.
// The running max may be stale by up to 2^8 (the final O / l uses the same reference);
// two column pairs in eight take 2^x from the FMA-pipe polynomial. Each thread loads its
// row of S in two 64-column halves: the max of the first half overlaps the load of the
// second (four quarters were slower).
#pragma once

#include "ptx.cuh"

namespace attn {
namespace enc1q {

// 64 columns of this warp's 32 TMEM lanes, left in flight (tc_wait_ld64 completes them)
__device__ __forceinline__ void tmem_ld64_async(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
                 : "r"(taddr)
                 : "memory");
}
// waits for the warp's TMEM loads; r is named so that no read of it moves above the wait
__device__ __forceinline__ void tc_wait_ld64(uint32_t (&r)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63]) :: "memory");
}

constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kD = 64;
constexpr int kThreads = 192;          // warps 0-3 softmax, 4 producer, 5 MMA issuer
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kStages = 2;
constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 128, kColP = 192;
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPolyEighths = 2;

constexpr int kQOff = 0;
constexpr int kKOff = kQOff + kTileBytes;
constexpr int kVOff = kKOff + kStages * kTileBytes;
constexpr int kBarOff = kVOff + kStages * kTileBytes;
// q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full, s_free, p_ready[4], pv_done,
// o_final, mma_done, count_ready, bias_full[S], bias_empty[S]
constexpr int kPChunks = kTileN / 32;   // P is written, and P.V issued, in 32-key chunks
constexpr int kNumBars = 1 + 4 * kStages + 6 + kPChunks + 2 * kStages;
constexpr int kMiscOff = kBarOff + kNumBars * 8;   // TMEM address, abort flag, live tile count
// with a key bias: per ring stage the tile's bias in log2 units (128 floats) and one word,
// the first -inf column when the tile is a prefix mask (zeros, then -inf), else -1
constexpr int kBiasOff = (kMiscOff + 16 + 15) & ~15;
constexpr int kBiasInfoOff = kBiasOff + kStages * kTileN * 4;
constexpr int kSmemBytes = kBiasInfoOff + kStages * 4 + 1024;

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

template <bool kHasBias>
__global__ void __launch_bounds__(kThreads, 2)
encoder_1q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out,
                  const float* __restrict__ key_bias, int H, int S, float scale_log2) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* k_full = q_full + 1;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* v_full = k_empty + kStages;
    uint64_t* v_empty = v_full + kStages;
    uint64_t* s_full = v_empty + kStages;
    uint64_t* s_free = s_full + 1;
    uint64_t* p_ready = s_free + 1;
    uint64_t* pv_done = p_ready + kPChunks;
    uint64_t* o_final = pv_done + 1;
    uint64_t* mma_done = o_final + 1;
    uint64_t* count_ready = mma_done + 1;
    uint64_t* bias_full = count_ready + 1;      // the producer has staged tile j's bias
    uint64_t* bias_empty = bias_full + kStages; // the softmax warps are done with it
    float* bias_s = reinterpret_cast<float*>(smem + kBiasOff);
    volatile int* bias_info = reinterpret_cast<volatile int*>(smem + kBiasInfoOff);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 4);
    // with a key bias: the key tiles that hold a kept key (the producer counts them while the
    // first copies fly and publishes the count through count_ready)
    volatile int* n_live_slot = reinterpret_cast<volatile int*>(smem + kMiscOff + 8);

    const int warp = threadIdx.x >> 5;
    const int bh = blockIdx.y;
    const int row0 = blockIdx.x * kTileM;
    const int n_kv_all = (S + kTileN - 1) / kTileN;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);    // one arrival per softmax warp
        for (int c = 0; c < kPChunks; ++c) mbar_init(&p_ready[c], 4);
        mbar_init(pv_done, 1);
        mbar_init(o_final, 1);
        mbar_init(mma_done, 1);
        mbar_init(count_ready, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bias_full[s], 1);
            mbar_init(&bias_empty[s], 4);   // one arrival per softmax warp
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
    pdl_launch_dependents();
    pdl_wait_predecessor();
    int issued_k = 0, issued_v = 0;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        bool ok = true;
        auto load_kv = [&](int j) {   // K and V tile j into ring stage j % kStages (lane 0)
            const int st = j % kStages;
            const uint32_t use = j / kStages;
            if (use > 0) ok = mbar_wait(&k_empty[st], (use - 1) & 1, abort_flag);
            if (!ok) return;
            mbar_arrive_expect_tx(&k_full[st], kTileBytes);
            tma_load_3d(smem + kKOff + st * kTileBytes, &tm_k, &k_full[st], 0, j * kTileN, bh);
            issued_k = j + 1;
            if (use > 0) ok = mbar_wait(&v_empty[st], (use - 1) & 1, abort_flag);
            if (!ok) return;
            mbar_arrive_expect_tx(&v_full[st], kTileBytes);
            tma_load_3d(smem + kVOff + st * kTileBytes, &tm_v, &v_full[st], 0, j * kTileN, bh);
            issued_v = j + 1;
        };
        if (lane_id() == 0) {
            mbar_arrive_expect_tx(q_full, kTileBytes);
            tma_load_3d(smem + kQOff, &tm_q, q_full, 0, row0, bh);
            load_kv(0);
        }
        __syncwarp();
        if constexpr (!kHasBias) {
            if (lane_id() == 0)
                for (int j = 1; j < n_kv_all && ok; ++j) load_kv(j);
        } else {
            const float* kb_row = key_bias + static_cast<size_t>(bh / H) * S;
            const int n_kv = live_key_tiles(kb_row, S);
            if (lane_id() == 0) {
                *n_live_slot = n_kv;
                mbar_arrive(count_ready);   // release: the count is visible to the waiters
            }
            // Tile j's bias into ring stage j % kStages, whole warp, four columns per lane:
            // in log2 units (-inf kept, a finite value clamped at -FLT_MAX so that its key
            // stays), and whether the tile is a prefix mask: zeros up to its first -inf
            // column, -inf from there on (no bias, or the end of a right-padded entry).
            auto stage_bias = [&](int j) -> bool {
                const int st = j % kStages;
                const uint32_t use = j / kStages;
                if (use > 0 && !mbar_wait_warp(&bias_empty[st], (use - 1) & 1, abort_flag)) return false;
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
                if (lane_id() == 0) mbar_arrive(&bias_full[st]);   // release: the stage is visible
                return true;
            };
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (ok) ok = stage_bias(0);
            for (int j = 1; j < n_kv && ok; ++j) {
                if (lane_id() == 0) load_kv(j);
                ok = __shfl_sync(0xffffffffu, ok, 0);   // lane 0's copies decide for the warp
                if (ok) ok = stage_bias(j);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane_id() == 0) {
            constexpr uint32_t idesc_qk = make_idesc(kTileM, kTileN, 1, 1, 0, 0);
            constexpr uint32_t idesc_pv = make_idesc(kTileM, kD, 1, 1, 0, 1);
            const uint64_t dq = smem_desc(smem_u32(smem + kQOff), 16, 1024);
            const uint64_t dk = smem_desc(smem_u32(smem + kKOff), 16, 1024);
            const uint64_t dv = smem_desc(smem_u32(smem + kVOff), kTileBytes, 1024);
            auto issue_qk = [&](int st) {
                const uint64_t ka = dk + static_cast<uint64_t>((st * kTileBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    mma_f16_ss(tmem_base + kColS, dq + 2 * kk, ka + 2 * kk, idesc_qk, kk > 0);
            };
            auto issue_pv = [&](int st, int c, bool acc) {   // keys 32 c .. 32 c + 31
                const uint64_t va = dv + static_cast<uint64_t>((st * kTileBytes) >> 4);
#pragma unroll
                for (int kk = 2 * c; kk < 2 * c + 2; ++kk)
                    mma_f16_ts(tmem_base + kColO, tmem_base + kColP + kk * 8,
                               va + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                               (acc || kk > 0) ? 1u : 0u);
            };
            bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&k_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_qk(0);
                tc_commit(s_full);
                tc_commit(&k_empty[0]);
            }
            int n_kv = n_kv_all;
            if constexpr (kHasBias) {
                if (ok) ok = mbar_wait(count_ready, 0, abort_flag);
                n_kv = *n_live_slot;
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                if (j + 1 < n_kv) {   // S(j+1) once the softmax has read S(j)
                    const int stn = (j + 1) % kStages;
                    ok = mbar_wait(s_free, j & 1, abort_flag) &&
                         mbar_wait(&k_full[stn], ((j + 1) / kStages) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_qk(stn);
                    tc_commit(s_full);
                    tc_commit(&k_empty[stn]);
                }
                const int st = j % kStages;
                ok = mbar_wait(&v_full[st], (j / kStages) & 1, abort_flag);
                for (int c = 0; c < kPChunks && ok; ++c) {   // each chunk as soon as it is in
                    ok = mbar_wait(&p_ready[c], j & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(st, c, j > 0);
                }
                if (!ok) break;
                tc_commit(pv_done);
                tc_commit(&v_empty[st]);
            }
            if (ok) tc_commit(o_final);
            tc_commit(mma_done);   // teardown waits for it on an abort
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax: one thread per row
        const int r = threadIdx.x;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tS = tmem_base + lane_off + kColS;
        const uint32_t tO = tmem_base + lane_off + kColO;
        const uint32_t tP = tmem_base + lane_off + kColP;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        int n_kv = n_kv_all;
        if constexpr (kHasBias) {
            ok = mbar_wait_warp(count_ready, 0, abort_flag);
            n_kv = *n_live_slot;
        }
        bool s_seen = false;   // S(j) already reported complete by an earlier look
        for (int j = 0; ok && j < n_kv; ++j) {
            if (!__all_sync(0xffffffffu, s_seen)) {
                ok = mbar_wait_warp(s_full, j & 1, abort_flag);
                if (!ok) break;
            }
            tc_fence_after();
            const int kv0 = j * kTileN;
            int valid = S - kv0;    // columns of this tile that take part (the rest are -inf)
            bool raw_path = true;   // scores taken as they are (no key bias on this tile)
            const float* bl = nullptr;
            if constexpr (kHasBias) {
                // the producer has staged this tile's bias: a prefix mask (zeros, then -inf)
                // is computed as without a bias with its -inf part masked like the columns
                // past S; any other tile adds the staged log2-unit bias to its scores
                const int stb = j % kStages;
                ok = mbar_wait_warp(&bias_full[stb], (j / kStages) & 1, abort_flag);
                if (!ok) break;
                const int info = bias_info[stb];
                raw_path = info >= 0;
                if (raw_path) {
                    valid = info;
                    __syncwarp();
                    if (lane_id() == 0) mbar_arrive(&bias_empty[stb]);
                } else {
                    bl = bias_s + stb * kTileN;
                }
            }
            uint32_t u[kTileN];
            uint32_t (&ua)[64] = *reinterpret_cast<uint32_t(*)[64]>(u);
            uint32_t (&ub)[64] = *reinterpret_cast<uint32_t(*)[64]>(u + 64);
            static_assert(kTileN == 128, "the row is loaded and maxed in two halves of 64");
            float mx[4];
            float m_tile;
            bool pv_seen = true;
            if (raw_path) {
                tmem_ld64_wait(tS, ua);
                tmem_ld64_async(tS + 64, ub);   // the second half lands while the first is maxed
                // raw scores (scale folded into the exponent); columns past S are -inf
                if (valid < 64) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (i >= valid) u[i] = __float_as_uint(-INFINITY);
                }
                // pairs first, then three-input maxes over groups of 8 columns
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    mx[e] = fmaxf(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
#pragma unroll
                for (int i = 8; i < 64; i += 8) {
                    mx[0] = fmax3(mx[0], __uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                    mx[1] = fmax3(mx[1], __uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
                    mx[2] = fmax3(mx[2], __uint_as_float(u[i + 4]), __uint_as_float(u[i + 5]));
                    mx[3] = fmax3(mx[3], __uint_as_float(u[i + 6]), __uint_as_float(u[i + 7]));
                }
                tc_wait_ld64(ub);
                tc_fence_before();     // S may be overwritten by QK(j+1) from here on
                __syncwarp();
                if (lane_id() == 0) mbar_arrive(s_free);
                // PV(j-1) was issued when P(j-1) was complete and has most likely finished:
                // look now, use the answer before P(j) is stored
                pv_seen = j == 0 || mbar_test(pv_done, (j - 1) & 1);
                if (valid < kTileN) {
#pragma unroll
                    for (int i = 64; i < kTileN; ++i)
                        if (i >= valid) u[i] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int i = 64; i < kTileN; i += 8) {
                    mx[0] = fmax3(mx[0], __uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                    mx[1] = fmax3(mx[1], __uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
                    mx[2] = fmax3(mx[2], __uint_as_float(u[i + 4]), __uint_as_float(u[i + 5]));
                    mx[3] = fmax3(mx[3], __uint_as_float(u[i + 6]), __uint_as_float(u[i + 7]));
                }
                m_tile = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * scale_log2;
            } else if constexpr (kHasBias) {
                tmem_ld64_wait(tS, ua);
                tmem_ld64_wait(tS + 64, ub);
                tc_fence_before();     // S may be overwritten by QK(j+1) from here on
                __syncwarp();
                if (lane_id() == 0) mbar_arrive(s_free);
                pv_seen = j == 0 || mbar_test(pv_done, (j - 1) & 1);
                // biased score in log2 units: one FMA per score against the staged bias
                // (-inf where the key is dropped or past S: the staged value is -inf there)
                mx[0] = mx[1] = mx[2] = mx[3] = -INFINITY;
#pragma unroll
                for (int i = 0; i < kTileN; i += 4) {
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
                if (lane_id() == 0) mbar_arrive(&bias_empty[j % kStages]);
                m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            }
            // log2-unit factor of the scores in u: the scale on the raw path, 1 on the biased one
            const float sc = raw_path ? scale_log2 : 1.f;
            const bool upd = m_tile > m_run + kRescaleThreshold;
            const float m_next = upd ? m_tile : m_run;
            const float m_use = (m_next == -INFINITY) ? 0.f : m_next;
            const float alpha = upd ? ex2_approx(m_run - m_use) : 1.f;
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kPChunks; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int kk = c * 16 + k;   // column pair index
                    const float2 sv = make_float2(__uint_as_float(u[2 * kk]), __uint_as_float(u[2 * kk + 1]));
                    const float2 x = __ffma2_rn(sv, make_float2(sc, sc), make_float2(-m_use, -m_use));
                    float2 pv;
                    // the polynomial also takes the -inf columns of a ragged tile: it clamps
                    // them to 2^-125, and as past S the V rows are zero-filled they add
                    // nothing to O (and less than an ulp to the row sum)
                    if ((kk & 7) < kPolyEighths) {
                        pv = exp2_poly2(x);
                        if constexpr (kHasBias) {   // a dropped key weighs exactly 0 (its V may hold anything finite)
                            if (x.x == -INFINITY) pv.x = 0.f;
                            if (x.y == -INFINITY) pv.y = 0.f;
                        }
                    } else {
                        pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    }
                    if (k & 1) acc1 = __fadd2_rn(acc1, pv);
                    else acc0 = __fadd2_rn(acc0, pv);
                    pk[k] = pack_bf16x2(pv.x, pv.y);
                }
                if (c == 0 && j > 0) {
                    // P and O are free once PV of the previous tile has completed; O is
                    // rescaled now, before any part of PV(j) can be issued
                    if (!__all_sync(0xffffffffu, pv_seen)) {
                        ok = mbar_wait_warp(pv_done, (j - 1) & 1, abort_flag);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, upd)) {
#pragma unroll 1
                        for (int h = 0; h < kD / 16; ++h) {
                            uint32_t w[16];
                            tmem_ld16_wait(tO + h * 16, w);
#pragma unroll
                            for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
                            tmem_st16(tO + h * 16, w);
                        }
                    }
                }
                if (c > 0) {   // chunk c - 1 (and the O rescale) is in TMEM: PV may read it
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane_id() == 0) mbar_arrive(&p_ready[c - 1]);
                }
                // QK(j+1) was issued when S(j) had been read: look now whether S(j+1) is in
                if (c == kPChunks - 1) s_seen = j + 1 < n_kv && mbar_test(s_full, (j + 1) & 1);
                tmem_st16(tP + c * 16, pk);
            }
            if (!ok) break;
            l_run = l_run * alpha + ((acc0.x + acc0.y) + (acc1.x + acc1.y));
            m_run = m_next;
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane_id() == 0) mbar_arrive(&p_ready[kPChunks - 1]);
        }
        if (ok) ok = mbar_wait_warp(o_final, 0, abort_flag);
        if (ok) {
            tc_fence_after();
            const int row = row0 + r;
            const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
            uint16_t* orow = out + (static_cast<size_t>(bh) * S + row) * kD;
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t w[32];
                tmem_ld32_wait(tO + c * 32, w);
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
        tc_wait_st();
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a bounded wait ran out: every started copy lands and every MMA completes before
        // TMEM is freed and the CTA exits
        if (warp == kProducerWarp && lane_id() == 0) {
            mbar_wait_drain(q_full, 0);
            for (int j = (issued_k > kStages ? issued_k - kStages : 0); j < issued_k; ++j)
                mbar_wait_drain(&k_full[j % kStages], (j / kStages) & 1);
            for (int j = (issued_v > kStages ? issued_v - kStages : 0); j < issued_v; ++j)
                mbar_wait_drain(&v_full[j % kStages], (j / kStages) & 1);
        }
        if (warp == kMmaWarp && lane_id() == 0) mbar_wait_drain(mma_done, 0);
        __syncwarp();
    }
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace enc1q
}  // namespace attn
