// decode_mma.cuh -- the GQA decode stream step with the query heads of a KV head packed
// into one tensor-core tile (sm_100a warp-level MMA), used in place of the CUDA-core
// stream kernel of decode.cuh for head_dim 128 / 256.
//
// What it computes: exactly decode_stream_kernel's partials -- for every (batch, kv
// head) pair a warp covers, the unnormalised o = sum_j 2^(x_j - m) v_j, m and l over
// its slice of the pair's live keys, x_j = scale log2(e) q . k_j + mask_j (log2 units);
// the same slices, slot numbering, scan and combine ("head_dim>128 (256/512) GQA
// Flash-Decode NKI Kernel for AWS Trainium": the query heads that share a KV head are
// packed onto the matmul tile, "Input contract"; the split over the key sequence is
// the page's "Future performance follow-on").
//
// How. The num_kv_groups (G <= 8) heads of a pair form the N = 8 side of an
// m16n8k16 MMA and 16 keys (two 8-key sub-tiles of the warp's slice that belong to
// the same pair) the M side, so neither operand is padded to 128:
//     S^T [16 keys x 8 heads]  = K [16 x D] . Q^T [D x 8]          (D / 16 MMAs)
//     O^T [D x 8 heads]       += V^T [D x 16] . P^T [16 x 8]        (D / 16 MMAs)
// Q^T stays in registers for the whole pair, O^T is the fp32 accumulator (D / 16 tiles
// of 4 registers per lane). Per key the warp issues about 4 MMA-side instructions
// instead of 2 G D / 32 fused multiply-adds per lane, so the instruction issue stays
// far below the HBM time for any G. K and V sub-tiles arrive by TMA in 128-byte
// swizzled boxes (8 keys x 64 lanes, rows past S_ctx zero-filled), which makes every
// ldmatrix of K (row-major A) and V (transposed A) free of bank conflicts. P^T goes
// from the S accumulator to the B operand through a 256-byte shared tile and one
// transposing ldmatrix. V rows of dead keys inside a live sub-tile are zeroed before
// the P.V MMA (an MMA would multiply their p = 0 with whatever they hold).
//
// Included by decode.cuh after the shared pieces (workspace, cursors, scan) and before
// the host-side dispatch.
#pragma once

namespace attn {
namespace dec {

template <int D>
struct MmaCfg {
    static constexpr int kWarps = 6;
    static constexpr int kPanels = D / 64;                     // 128-byte swizzle panels per row
    static constexpr int kPanelBytes = 16 * 128;               // 16 keys x 128 bytes
    static constexpr int kHalfBytes = kPanels * kPanelBytes;   // K (or V) of one 16-key stage
    static constexpr int kStageBytes = 2 * kHalfBytes;         // K then V
    static constexpr int kStages = (D == 128) ? 4 : 2;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRingOff = 0;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kZeroOff = kRingOff + kRingBytes;                 // 1 KB of zeros
    static constexpr int kPtOff = kZeroOff + 1024;                         // [warp] P^T tile 256 B
    static constexpr int kMaskOff = kPtOff + kWarps * 256;                 // [warp][stage][16] fp32
    static constexpr int kInfoOff = kMaskOff + kWarps * kStages * 64;      // [warp][stage] int4
    static constexpr int kBarOff = kInfoOff + kWarps * kStages * 16;       // [warp][stage][K, V]
    static constexpr int kMiscOff = kBarOff + kWarps * kStages * 2 * 8;    // abort flag
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;                // + alignment slack
    static_assert(kWarps * 1 * 148 <= Cfg<D>::kMaxWarpsTotal, "slots sized for the CUDA-core path");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1) : "r"(addr));
}
// D = A (16x16, row) . B (16x8, col) + C, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared address of 16-byte chunk `chunk` (8 lanes of D) of row `r` (0..15) of a 16-key
// stage half in the 128-byte swizzle the TMA writes: panel chunk / 8, chunk index XOR
// (row mod 8) inside the 128-byte row.
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t base, int r, int chunk) {
    return base + (chunk >> 3) * MmaCfg<D>::kPanelBytes + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
}

template <int D, int G>
__global__ void __launch_bounds__(MmaCfg<D>::kThreads, 1)
decode_stream_mma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const uint16_t* __restrict__ q, Workspace ws, int B, int Hkv, int S_ctx,
                         float scale_log2) {
    using C = MmaCfg<D>;
    constexpr int kWarps = C::kWarps;
    constexpr int S = C::kStages;
    constexpr int kKSteps = D / 16;
    static_assert(G >= 1 && G <= 8, "up to 8 heads share a kv head");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;     // MMA fragment coordinates: group, thread in group
    const int n_sub = num_sub_tiles(S_ctx);
    uint8_t* ring_p = smem + C::kRingOff + warp * S * C::kStageBytes;
    const uint32_t ring = smem_u32(ring_p);
    const uint32_t zero = smem_u32(smem + C::kZeroOff);
    uint8_t* pt = smem + C::kPtOff + warp * 256;
    float* smask = reinterpret_cast<float*>(smem + C::kMaskOff) + warp * S * 16;
    int4* info = reinterpret_cast<int4*>(smem + C::kInfoOff) + warp * S;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kBarOff) + warp * S * 2;   // [stage][K, V]

    if (tid == 0) {
        for (int s = 0; s < kWarps * S * 2; ++s)
            mbar_init(reinterpret_cast<uint64_t*>(smem + C::kBarOff) + s, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    for (int i = tid; i < 256; i += C::kThreads) reinterpret_cast<uint32_t*>(smem + C::kZeroOff)[i] = 0u;
    __syncthreads();
    pdl_wait_predecessor();   // the scan kernel's counts, lists and compact mask are complete
    pdl_launch_dependents();

    // ---- this warp's slice of the item sequence (as in decode_stream_kernel)
    const int Pw = gridDim.x * kWarps, w = blockIdx.x * kWarps + warp;
    const int T = count_sums(ws.counts, B, 0, lane).total * Hkv;
    if (T == 0) return;
    const int c = (T + Pw - 1) / Pw;
    if (static_cast<long long>(w) * c >= T) return;
    const int lo = w * c;
    const int n = min(c, T - lo);

    // ---- issue side: steps of one or two consecutive items of one (b, g) pair
    Cursor wcur = cursor_at(ws.counts, B, Hkv, lo, lane);   // cursor of item wbase
    int wbase = 0;
    int my_sub = 0, my_bg = -1, my_slot = 0, my_idx = 0;
    auto fill_window = [&]() {
        my_bg = -1;
        if (wbase + lane < n) {
            const Cursor cc = cursor_advance(wcur, lane, ws.counts, Hkv);
            my_idx = cc.b * n_sub + cc.i;
            my_sub = ws.lists[my_idx];
            my_bg = cc.b * Hkv + cc.g;
            my_slot = w + Hkv * cc.nzb + cc.g;
        }
    };
    fill_window();
    int next_x = 0;                 // first item of the next step to issue
    int issued_k = 0, issued_v = 0; // steps whose K / V copies were started
    int pend_bg = 0, pend_k0a = 0, pend_k0b = 0, pend_n = 0;   // V half still to be issued (lane 0)
    constexpr uint32_t kItemBytes = C::kPanels * 1024;   // one 8-key box per panel
    // Issue the K half (and the mask) of step `t` starting at item next_x; whole warp calls.
    auto issue_k = [&](int t) {
        if (next_x - wbase > 30) {   // keep items x and x + 1 inside the window
            const int adv = next_x - wbase;
            wcur = cursor_advance(wcur, adv, ws.counts, Hkv);
            wbase += adv;
            fill_window();
        }
        const int L = next_x - wbase;
        const int sub0 = __shfl_sync(0xffffffffu, my_sub, L);
        const int bg0 = __shfl_sync(0xffffffffu, my_bg, L);
        const int slot0 = __shfl_sync(0xffffffffu, my_slot, L);
        const int idx0 = __shfl_sync(0xffffffffu, my_idx, L);
        const int sub1 = __shfl_sync(0xffffffffu, my_sub, L + 1);
        const int bg1 = __shfl_sync(0xffffffffu, my_bg, L + 1);
        const int idx1 = __shfl_sync(0xffffffffu, my_idx, L + 1);
        const int cnt = (next_x + 1 < n && bg1 == bg0) ? 2 : 1;
        next_x += cnt;
        if (lane == 0) {
            const int st = t % S;
            uint8_t* kdst = ring_p + st * C::kStageBytes;
            info[st] = make_int4(cnt, slot0, bg0, 0);
            pend_bg = bg0;
            pend_k0a = sub0 * kSubKeys;
            pend_k0b = sub1 * kSubKeys;
            pend_n = cnt;
            mbar_arrive_expect_tx(&bar[2 * st], cnt * (kItemBytes + kSubKeys * 4));
            for (int it = 0; it < cnt; ++it) {
                bulk_load(smask + st * 16 + it * 8, ws.maskc + static_cast<size_t>(it ? idx1 : idx0) * kSubKeys,
                          kSubKeys * 4, &bar[2 * st]);
                for (int p = 0; p < C::kPanels; ++p)
                    tma_load_3d(kdst + p * C::kPanelBytes + it * 1024, &tm_k, &bar[2 * st], p * 64,
                                it ? pend_k0b : pend_k0a, bg0);
            }
            issued_k = t + 1;
        }
        __syncwarp();   // info and the pending V description are visible to the whole warp
    };
    auto issue_v = [&](int t) {   // V half of step t, after issue_k(t) (lane 0 only)
        const int st = t % S;
        uint8_t* vdst = ring_p + st * C::kStageBytes + C::kHalfBytes;
        mbar_arrive_expect_tx(&bar[2 * st + 1], pend_n * kItemBytes);
        for (int it = 0; it < pend_n; ++it)
            for (int p = 0; p < C::kPanels; ++p)
                tma_load_3d(vdst + p * C::kPanelBytes + it * 1024, &tm_v, &bar[2 * st + 1], p * 64,
                            it ? pend_k0b : pend_k0a, pend_bg);
        issued_v = t + 1;
    };
    int n_steps_issued = 0;
    for (int t = 0; t < S && next_x < n; ++t) {
        issue_k(t);
        if (lane == 0) issue_v(t);
        ++n_steps_issued;
    }

    // ---- compute side
    uint32_t qb[kKSteps][2];   // Q^T as the B operand: lane holds head gq, lanes 2 tq(+1)(+8)
    float o[kKSteps][4];       // O^T accumulator: d = 16 i + gq (+8), heads 2 tq, 2 tq + 1
    float m_run[2], l_run[2];  // heads 2 tq, 2 tq + 1
    int cur_slot = -1;
    auto flush = [&](int slot) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 2 * tq + e;
            if (h < G) {
                float* dst = ws.o + (static_cast<size_t>(slot) * G + h) * D;
#pragma unroll
                for (int i = 0; i < kKSteps; ++i) {
                    dst[16 * i + gq] = o[i][e];
                    dst[16 * i + gq + 8] = o[i][2 + e];
                }
                if (gq == 0) {
                    ws.m[static_cast<size_t>(slot) * G + h] = m_run[e];
                    ws.l[static_cast<size_t>(slot) * G + h] = l_run[e];
                }
            }
        }
    };
    bool ok = true;
    int t = 0;
    for (; t < n_steps_issued && ok; ++t) {
        const int st = t % S;
        const uint32_t ph = (t / S) & 1;
        ok = mbar_wait_warp(&bar[2 * st], ph, abort_flag);
        if (!ok) break;
        const int4 inf = info[st];
        const int cnt = inf.x;
        if (inf.y != cur_slot) {   // a new (b, g) pair: close the previous one, load q
            if (cur_slot >= 0) flush(cur_slot);
            cur_slot = inf.y;
            const uint16_t* qh = q + (static_cast<size_t>(inf.z) * G + gq) * D;
#pragma unroll
            for (int i = 0; i < kKSteps; ++i) {
                qb[i][0] = gq < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * i + 2 * tq) : 0u;
                qb[i][1] = gq < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * i + 8 + 2 * tq) : 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
            }
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
        }
        // mask of keys gq and gq + 8 (log2 units; -inf dead, and the absent second item)
        const float mk0 = smask[st * 16 + gq];
        const float mk1 = cnt == 2 ? smask[st * 16 + 8 + gq] : -INFINITY;
        // dead keys of the live items (bit r = key r): their V rows are zeroed below
        const uint32_t dead = __ballot_sync(0xffffffffu, lane < 8 * cnt && smask[st * 16 + (lane & 15)] == -INFINITY);
        const uint32_t kbase = ring + st * C::kStageBytes;
        const uint32_t vbase = kbase + C::kHalfBytes;
        // ---- S^T = K Q^T: A rows 0-7 item 0, rows 8-15 item 1 (or zeros)
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int mi = lane >> 3, r = lane & 7;            // ldmatrix: matrix, row
            const int row = r + 8 * (mi & 1);
            const bool use_zero = (mi & 1) && cnt == 1;
#pragma unroll
            for (int i = 0; i < kKSteps; ++i) {
                uint32_t a[4];
                const int chunk = 2 * i + (mi >> 1);
                ldsm_x4(use_zero ? zero + r * 128 : swz<D>(kbase, row, chunk), a);
                mma_16816(s, a, qb[i][0], qb[i][1]);
            }
        }
        __syncwarp();
        // K, the mask and the info of this stage are consumed: refill them with the next step
        if (next_x < n) {
            issue_k(n_steps_issued);
            ++n_steps_issued;
        }
        // ---- online softmax per head column over the 16 keys
        const float x0 = mk0 == -INFINITY ? -INFINITY : fmaf(s[0], scale_log2, mk0);
        const float x1 = mk0 == -INFINITY ? -INFINITY : fmaf(s[1], scale_log2, mk0);
        const float x2 = mk1 == -INFINITY ? -INFINITY : fmaf(s[2], scale_log2, mk1);
        const float x3 = mk1 == -INFINITY ? -INFINITY : fmaf(s[3], scale_log2, mk1);
        float mt[2] = {fmaxf(x0, x2), fmaxf(x1, x3)};
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mt[0] = fmaxf(mt[0], __shfl_xor_sync(0xffffffffu, mt[0], off));
            mt[1] = fmaxf(mt[1], __shfl_xor_sync(0xffffffffu, mt[1], off));
        }
        float alpha[2], mu[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float mn = fmaxf(m_run[e], mt[e]);
            mu[e] = (mn == -INFINITY) ? 0.f : mn;
            alpha[e] = ex2_approx(m_run[e] - mu[e]);
            m_run[e] = mn;
        }
        const float p0 = ex2_approx(x0 - mu[0]), p1 = ex2_approx(x1 - mu[1]);
        const float p2 = ex2_approx(x2 - mu[0]), p3 = ex2_approx(x3 - mu[1]);
        float ps[2] = {p0 + p2, p1 + p3};
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            ps[0] += __shfl_xor_sync(0xffffffffu, ps[0], off);
            ps[1] += __shfl_xor_sync(0xffffffffu, ps[1], off);
        }
        l_run[0] = l_run[0] * alpha[0] + ps[0];
        l_run[1] = l_run[1] * alpha[1] + ps[1];
        // P^T through shared memory: [key][head] bf16, then one transposing ldmatrix
        *reinterpret_cast<uint32_t*>(pt + gq * 16 + tq * 4) = pack_bf16x2(p0, p1);
        *reinterpret_cast<uint32_t*>(pt + (gq + 8) * 16 + tq * 4) = pack_bf16x2(p2, p3);
        __syncwarp();
        uint32_t pb0, pb1;
        ldsm_x2_t(smem_u32(pt) + (lane & 15) * 16, pb0, pb1);
        // rescale O^T if a head's running max moved
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
            for (int i = 0; i < kKSteps; ++i) {
                o[i][0] *= alpha[0];
                o[i][1] *= alpha[1];
                o[i][2] *= alpha[0];
                o[i][3] *= alpha[1];
            }
        }
        if (!mbar_wait_warp(&bar[2 * st + 1], ph, abort_flag)) {
            ok = false;
            break;
        }
        // dead keys of live items: zero their V rows (the MMA multiplies p = 0 by them)
        if (dead) {
            uint32_t bits = dead;
            while (bits) {
                const int r = __ffs(bits) - 1;
                bits &= bits - 1;
                for (int ch = lane; ch < D / 8; ch += 32)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(swz<D>(vbase, r, ch)),
                                 "r"(0u)
                                 : "memory");
            }
            __syncwarp();
        }
        // ---- O^T += V^T P^T: A = V^T via transposing ldmatrix (rows 8-15 item 1 or zeros)
        {
            const int mi = lane >> 3, r = lane & 7;
            const int key = r + 8 * (mi >> 1);                 // matrices: (k0-7,d0-7) (k0-7,d8-15) (k8-15,d0-7) (k8-15,d8-15)
            const bool use_zero = (mi >> 1) && cnt == 1;
#pragma unroll
            for (int i = 0; i < kKSteps; ++i) {
                uint32_t a[4];
                const int chunk = 2 * i + (mi & 1);
                ldsm_x4_t(use_zero ? zero + r * 128 : swz<D>(vbase, key, chunk), a);
                // A fragment order: a0 (d 0-7, k 0-7), a1 (d 8-15, k 0-7), a2 (d 0-7, k 8-15), a3 (d 8-15, k 8-15)
                mma_16816(o[i], a, pb0, pb1);
            }
        }
        // V of this stage is consumed; zeros written through the generic proxy must be
        // ordered before the next TMA write into the stage
        if (dead) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && t + S < n_steps_issued) issue_v(t + S);
    }
    if (ok) {
        if (cur_slot >= 0) flush(cur_slot);
    } else if (lane == 0) {   // let every copy this warp started land before the CTA exits
        for (int x = max(0, issued_k - S); x < issued_k; ++x)
            mbar_wait_drain(&bar[2 * (x % S)], (x / S) & 1);
        for (int x = max(0, issued_v - S); x < issued_v; ++x)
            mbar_wait_drain(&bar[2 * (x % S) + 1], (x / S) & 1);
    }
}

}  // namespace dec
}  // namespace attn
