// decode.cuh -- single-token GQA flash-decode for sm_100a.
//
// What it computes ("head_dim>128 (256/512) GQA Flash-Decode NKI Kernel for
// AWS Trainium", "Input contract"): for every batch entry b and query head h,
//   out[b,h] = softmax(scale * q[b,h] K[b,g]^T + attn_mask[b]) V[b,g],
//   g = h / num_kv_groups, S_q = 1, head_dim D in {128, 256, 512}.
//
// How. Decode is bound by HBM bandwidth (each K/V byte serves only
// num_kv_groups query heads), so the tensor cores stay idle and the design is
// about streaming the live K/V once, at full bandwidth, with every SM busy
// until the end whatever the mix of context lengths. Three launches on the
// caller's stream:
//   1. decode_scan_kernel (one CTA per batch entry) turns the additive mask
//      into the list of live 8-key sub-tiles (a key is live when its mask is
//      not -inf and it lies before S_ctx) and a compact copy of their mask
//      values in log2 units; sub-tiles with no live key are never read;
//   2. decode_stream_kernel runs exactly one wave of warps. The live sub-tiles
//      of all (batch, kv head) pairs form one sequence of T items, ordered by
//      (b, g, list position); warp w takes the contiguous slice
//      [w c, (w + 1) c), c = ceil(T / warps), so every warp streams the same
//      number of bytes (the page's "multi-program dispatch" follow-on, with
//      the work split evenly instead of per context). A warp pulls each
//      sub-tile's K and V rows with bulk async copies (cp.async.bulk) into a
//      private shared-memory ring and keeps the running max / sum / numerator
//      of the num_kv_groups query heads that share the kv head (the pages' GQA
//      head packing, as data reuse); q . k partial sums are reduced with a
//      transposed butterfly (one shuffle per (key, head) pair). When its slice
//      crosses from one pair to the next, the warp writes the finished pair's
//      unnormalised partial (o, m, l) and starts afresh. Warps never wait for
//      one another;
//   3. decode_combine_kernel finds the partials of each (batch, kv head) from
//      the counts alone and applies the log-sum-exp rule.
// Kernels 2 and 3 are programmatic dependents of their predecessors (PDL), so
// their set-up overlaps the previous kernel's tail.
//
// Partial slots. With J(b, g) = Hkv * (number of non-empty batch entries before
// b) + g, the index of a non-empty pair among all non-empty pairs, warp w's
// partial of pair (b, g) goes to slot w + J(b, g). One warp's pairs have
// increasing J, and a warp's first pair is at least the previous warp's last,
// so slots never collide; a pair covered by warps w0..w1 owns the contiguous
// slots w0 + J .. w1 + J. At most (warps + B * Hkv) slots are used.
//
// Scores are kept in log2 units (scale * log2 e folded into q, mask * log2 e
// in the scan) so every exponential is one ex2 instruction.
#pragma once

#include "ptx.cuh"
#include "tmap.cuh"

namespace attn {
namespace dec {

constexpr int kSubKeys = 8;                  // keys per sub-tile (one ring stage)
constexpr int kMaxGroups = 8;
constexpr int kScanThreads = 1024;
constexpr int kSms = 148;                    // one wave is sized for at most this many SMs
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int num_sub_tiles(int S_ctx) { return (S_ctx + kSubKeys - 1) / kSubKeys; }
inline size_t round256(size_t x) { return ((x + 255) / 256) * 256; }

template <int D>
struct Cfg {
    // warps per CTA and ring stages per warp: ~96 KB of ring per CTA (two CTAs per SM)
    // for D <= 256; D = 512 uses 4 warps x 2 stages (128 KB, one CTA per SM)
    static constexpr int kWarps = (D == 512) ? 4 : 6;
    static constexpr int kCtasPerSm = (D == 512) ? 1 : 2;
    static constexpr int kMaxWarpsTotal = kSms * kCtasPerSm * kWarps;   // partial slots per pair sweep
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kRowBytes = D * 2;
    static constexpr int kSubBytes = kSubKeys * kRowBytes;       // K (or V) rows of one sub-tile
    static constexpr int kStageBytes = 2 * kSubBytes;            // K then V
    static constexpr int kStages = (D == 128) ? 4 : 2;           // per warp
    static constexpr int kEPL = D / 32;                          // elements of D per lane
    static constexpr int kRingOff = 0;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kMaskOff = kRingOff + kRingBytes;                 // [warp][stage][8] fp32
    static constexpr int kInfoOff = kMaskOff + kWarps * kStages * 32;      // [warp][stage] int4
    static constexpr int kScrOff = kInfoOff + kWarps * kStages * 16;       // [warp]: P [G][8], alpha [G]
    static constexpr int kScrFloats = kMaxGroups * kSubKeys + kMaxGroups;
    static constexpr int kBarOff = kScrOff + kWarps * kScrFloats * 4;      // [warp][stage][K, V]
    static constexpr int kMiscOff = kBarOff + kWarps * kStages * 2 * 8;    // abort flag
    static constexpr int kSmemBytes = kMiscOff + 16;
};

inline int max_warps_total(int D) {
    switch (D) {
        case 128: return Cfg<128>::kMaxWarpsTotal;
        case 256: return Cfg<256>::kMaxWarpsTotal;
        default: return Cfg<512>::kMaxWarpsTotal;
    }
}

// Workspace: counts [B] int32; live lists [B][n_sub] int32; compact mask
// [B][n_sub][8] fp32; partials o [slot][G][D], m and l [slot][G] fp32.
struct Workspace {
    int* counts;
    int* lists;
    float* maskc;
    float* o;
    float* m;
    float* l;
};

inline size_t num_slots(int B, int Hkv, int D) {
    return static_cast<size_t>(max_warps_total(D)) + static_cast<size_t>(B) * Hkv;
}

inline size_t workspace_bytes(int B, int Hq, int Hkv, int S_ctx, int D) {
    const size_t G = static_cast<size_t>(Hq / Hkv);
    const size_t items = static_cast<size_t>(B) * num_sub_tiles(S_ctx);
    const size_t slots = num_slots(B, Hkv, D);
    return round256(static_cast<size_t>(B) * 4) + round256(items * 4) + round256(items * 32) +
           round256(slots * G * D * 4) + 2 * round256(slots * G * 4);
}

inline Workspace carve_workspace(void* base, int B, int Hq, int Hkv, int S_ctx, int D) {
    const size_t G = static_cast<size_t>(Hq / Hkv);
    const size_t items = static_cast<size_t>(B) * num_sub_tiles(S_ctx);
    const size_t slots = num_slots(B, Hkv, D);
    uint8_t* p = static_cast<uint8_t*>(base);
    Workspace w;
    w.counts = reinterpret_cast<int*>(p);
    p += round256(static_cast<size_t>(B) * 4);
    w.lists = reinterpret_cast<int*>(p);
    p += round256(items * 4);
    w.maskc = reinterpret_cast<float*>(p);
    p += round256(items * 32);
    w.o = reinterpret_cast<float*>(p);
    p += round256(slots * G * D * 4);
    w.m = reinterpret_cast<float*>(p);
    p += round256(slots * G * 4);
    w.l = reinterpret_cast<float*>(p);
    return w;
}

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

__device__ __forceinline__ int warp_sum(int x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}


// Sums over the live counts, computed by a whole warp (lane-strided, then reduced):
// total = sum_b counts[b]; before = sum_{b' < b} counts[b'];
// nz_before = number of b' < b with counts[b'] > 0.
struct CountSums {
    int total, before, nz_before;
};
template <bool kL2Only = false>
__device__ __forceinline__ CountSums count_sums(const int* counts, int B, int b, int lane) {
    int t = 0, bf = 0, nz = 0;
    for (int i = lane; i < B; i += 32) {
        const int c = kL2Only ? __ldcg(counts + i) : counts[i];
        t += c;
        if (i < b) {
            bf += c;
            nz += c > 0;
        }
    }
    return {warp_sum(t), warp_sum(bf), warp_sum(nz)};
}

// ---------------------------------------------------------------- 1. scan
__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const float* __restrict__ mask, int S_ctx, Workspace ws) {
    __shared__ int warp_n[kScanThreads / 32];
    pdl_launch_dependents();   // the stream kernel may set up; it waits for this grid itself
    // Pull this row of the mask into L2 while the previous kernel finishes (a prefetch
    // only warms L2, the point of coherence, so it cannot return stale data).
    if (mask)
        for (int off = threadIdx.x * 32; off < S_ctx; off += kScanThreads * 32)
            prefetch_l2(mask + static_cast<size_t>(blockIdx.x) * S_ctx + off);
    // whatever ran before on the stream (the previous call's combine kernel reading the
    // counts, or the caller's kernel writing the mask) has finished and its writes are visible
    pdl_wait_predecessor();
    const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_sub = num_sub_tiles(S_ctx);
    const size_t row = static_cast<size_t>(b) * n_sub;
    int n = 0;
    for (int base = 0; base < n_sub; base += kScanThreads) {
        const int st = base + tid;
        float mv[kSubKeys];
        bool live = false;
#pragma unroll
        for (int kk = 0; kk < kSubKeys; ++kk) {
            const int key = st * kSubKeys + kk;
            // liveness is decided on the stored value: only -inf removes a key. A finite mask
            // value is clamped after the change to log2 units, so that large negative fills
            // (e.g. -FLT_MAX) stay finite and keep their key, as the definition says.
            float x = -INFINITY;
            if (st < n_sub && key < S_ctx) {
                const float mraw = mask ? mask[static_cast<size_t>(b) * S_ctx + key] : 0.f;
                if (mraw != -INFINITY) x = fmaxf(mraw * kLog2e, -FLT_MAX);
            }
            mv[kk] = x;
            live |= (x != -INFINITY);
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, live);
        if (lane == 0) warp_n[warp] = __popc(bal);
        __syncthreads();
        int before = n, total = 0;
        for (int w = 0; w < kScanThreads / 32; ++w) {
            const int c = warp_n[w];
            before += (w < warp) ? c : 0;
            total += c;
        }
        if (live) {
            const size_t pos = row + before + __popc(bal & ((1u << lane) - 1u));
            ws.lists[pos] = st;
            float4* dst = reinterpret_cast<float4*>(ws.maskc + pos * kSubKeys);
            dst[0] = make_float4(mv[0], mv[1], mv[2], mv[3]);
            dst[1] = make_float4(mv[4], mv[5], mv[6], mv[7]);
        }
        n += total;
        __syncthreads();
    }
    if (tid == 0) ws.counts[b] = n;
}

// ---------------------------------------------------------------- 2. stream
// Position in the item sequence: pair (b, g), list position i, counts[b] = cb,
// nzb = number of non-empty batch entries before b.
struct Cursor {
    int b, g, i, cb, nzb;
};

// The cursor `steps` items after c (the item must exist).
__device__ __forceinline__ Cursor cursor_advance(Cursor c, int steps, const int* counts, int Hkv) {
    int x = c.g * c.cb + c.i + steps;   // offset within batch entry c.b's items
    while (x >= Hkv * c.cb) {
        x -= Hkv * c.cb;
        ++c.nzb;
        do {
            c.cb = counts[++c.b];
        } while (c.cb == 0);
    }
    c.g = x / c.cb;
    c.i = x - c.g * c.cb;
    return c;
}

// The cursor of item x (0 <= x < Hkv * sum(counts)), found by the whole warp.
__device__ __forceinline__ Cursor cursor_at(const int* counts, int B, int Hkv, int x, int lane) {
    int base = 0, nz = 0;
    Cursor c{0, 0, 0, 0, 0};
    for (int b0 = 0; b0 < B; b0 += 32) {
        const int cb = (b0 + lane < B) ? counts[b0 + lane] : 0;
        const int items = cb * Hkv;
        int incl = items;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, base + incl > x);
        const uint32_t nzbal = __ballot_sync(0xffffffffu, cb > 0);
        if (hit) {
            const int L = __ffs(hit) - 1;
            const int cbL = __shfl_sync(0xffffffffu, cb, L);
            const int pre = base + __shfl_sync(0xffffffffu, incl - items, L);
            const int off = x - pre;
            c.b = b0 + L;
            c.cb = cbL;
            c.g = off / cbL;
            c.i = off - c.g * cbL;
            c.nzb = nz + __popc(nzbal & ((1u << L) - 1u));
            return c;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
        nz += __popc(nzbal);
    }
    return c;
}

template <int D, int G>
__global__ void __launch_bounds__(Cfg<D>::kThreads)
decode_stream_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                     const uint16_t* __restrict__ v, Workspace ws, int B, int Hkv, int S_ctx,
                     float scale_log2) {
    using C = Cfg<D>;
    constexpr int kWarps = C::kWarps;
    constexpr int S = C::kStages;
    constexpr int kHeadsPerPass = G < 4 ? G : 4;       // N = 8 * heads <= 32 values per butterfly
    constexpr int kPasses = G / kHeadsPerPass;
    constexpr int kN = kSubKeys * kHeadsPerPass;
    constexpr int kBase = 32 / kN;                      // lanes sharing one value index
    extern __shared__ __align__(128) uint8_t smem[];
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_sub = num_sub_tiles(S_ctx);
    uint8_t* ring = smem + C::kRingOff + warp * S * C::kStageBytes;
    float* smask = reinterpret_cast<float*>(smem + C::kMaskOff) + warp * S * kSubKeys;
    int4* info = reinterpret_cast<int4*>(smem + C::kInfoOff) + warp * S;
    float* scr = reinterpret_cast<float*>(smem + C::kScrOff) + warp * C::kScrFloats;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kBarOff) + warp * S * 2;   // [stage][K, V]

    if (tid == 0) {
        for (int s = 0; s < kWarps * S * 2; ++s)
            mbar_init(reinterpret_cast<uint64_t*>(smem + C::kBarOff) + s, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait_predecessor();   // the scan kernel's counts, lists and compact mask are complete
    // The combine kernel may set up from here on: the scan has completed, so the counts it
    // reads before its own wait are final.
    pdl_launch_dependents();

    // ---- this warp's slice of the item sequence
    const int Pw = gridDim.x * kWarps, w = blockIdx.x * kWarps + warp;
    const int T = count_sums(ws.counts, B, 0, lane).total * Hkv;
    if (T == 0) return;
    const int c = (T + Pw - 1) / Pw;
    if (static_cast<long long>(w) * c >= T) return;
    const int lo = w * c;
    const int n = min(c, T - lo);

    // ---- issue side. A window of 32 items is described lane-parallel (lane L: item
    // wbase + L), so the list entries of a whole window arrive in one round trip.
    Cursor wcur = cursor_at(ws.counts, B, Hkv, lo, lane);   // cursor of item wbase
    int wbase = 0;
    int my_sub = 0, my_bg = 0, my_slot = 0, my_idx = 0;     // this lane's item of the window
    auto fill_window = [&]() {
        if (wbase + lane < n) {
            const Cursor c = cursor_advance(wcur, lane, ws.counts, Hkv);
            my_idx = c.b * n_sub + c.i;
            my_sub = ws.lists[my_idx];
            my_bg = c.b * Hkv + c.g;
            my_slot = w + Hkv * c.nzb + c.g;
        }
    };
    fill_window();
    size_t pend_src = 0;       // K/V row offset of the item whose V half is still to be issued
    uint32_t pend_bytes = 0;
    int issued_k = 0, issued_v = 0;
    auto issue_k = [&](int x) {   // item x of the slice -> stage x % S (whole warp calls)
        if (x - wbase >= 32) {
            wcur = cursor_advance(wcur, 32, ws.counts, Hkv);
            wbase += 32;
            fill_window();
        }
        const int L = x - wbase;
        const int sub = __shfl_sync(0xffffffffu, my_sub, L);
        const int bg = __shfl_sync(0xffffffffu, my_bg, L);
        const int slot = __shfl_sync(0xffffffffu, my_slot, L);
        const int idx = __shfl_sync(0xffffffffu, my_idx, L);
        if (lane == 0) {
            const int st = x % S;
            const int kk0 = sub * kSubKeys;
            const int rows = min(kSubKeys, S_ctx - kk0);
            info[st] = make_int4(kk0, rows, slot, bg);
            pend_src = static_cast<size_t>(bg) * S_ctx + kk0;
            pend_bytes = static_cast<uint32_t>(rows) * C::kRowBytes;
            mbar_arrive_expect_tx(&bar[2 * st], pend_bytes + kSubKeys * 4);
            bulk_load(smask + st * kSubKeys, ws.maskc + static_cast<size_t>(idx) * kSubKeys,
                      kSubKeys * 4, &bar[2 * st]);
            bulk_load(ring + st * C::kStageBytes, k + pend_src * D, pend_bytes, &bar[2 * st]);
            issued_k = x + 1;
        }
    };
    auto issue_v = [&](int x) {   // V half of item x, after issue_k(x) (lane 0 only)
        const int st = x % S;
        mbar_arrive_expect_tx(&bar[2 * st + 1], pend_bytes);
        bulk_load(ring + st * C::kStageBytes + C::kSubBytes, v + pend_src * D, pend_bytes,
                  &bar[2 * st + 1]);
        issued_v = x + 1;
    };
    for (int x = 0; x < n && x < S; ++x) {
        issue_k(x);
        if (lane == 0) issue_v(x);
    }

    // ---- compute side (all lanes)
    const int idx_me = lane / kBase;                    // value index held after the butterfly
    const int hh_me = idx_me / kSubKeys, kk_me = idx_me % kSubKeys;
    float qr[G][C::kEPL];
    float o[G][C::kEPL];
    float m_run[G], l_run[G];
    int cur_slot = -1;
    auto flush = [&](int slot) {   // unnormalised partial of the finished pair
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float4* dst = reinterpret_cast<float4*>(ws.o + (static_cast<size_t>(slot) * G + h) * D +
                                                    lane * C::kEPL);
#pragma unroll
            for (int e = 0; e < C::kEPL; e += 4)
                dst[e / 4] = make_float4(o[h][e], o[h][e + 1], o[h][e + 2], o[h][e + 3]);
        }
        if (lane == 0)
#pragma unroll
            for (int h = 0; h < G; ++h) {
                ws.m[static_cast<size_t>(slot) * G + h] = m_run[h];
                ws.l[static_cast<size_t>(slot) * G + h] = l_run[h];
            }
    };
    bool ok = true;

    for (int u = 0; u < n; ++u) {
        const int st = u % S;
        const uint32_t ph = (u / S) & 1;
        ok = mbar_wait_warp(&bar[2 * st], ph, abort_flag);
        if (!ok) break;
        const int4 inf = info[st];
        const float mv = smask[st * kSubKeys + kk_me];
        // keys of this sub-tile that take part: bit kk * kBase is set when key kk is live
        // (mask not -inf; keys past S_ctx carry -inf). Taken now, because the stage's mask
        // slot is refilled before the P.V step below.
        const uint32_t live_bits = __ballot_sync(0xffffffffu, mv != -INFINITY);
        if (inf.z != cur_slot) {   // a new (b, g) pair: close the previous one, load q
            if (cur_slot >= 0) flush(cur_slot);
            cur_slot = inf.z;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint16_t* qh = q + (static_cast<size_t>(inf.w) * G + h) * D + lane * C::kEPL;
                uint32_t wq[C::kEPL / 2];
                load_bf16_words<C::kEPL>(qh, wq);
#pragma unroll
                for (int i = 0; i < C::kEPL / 2; ++i) {
                    qr[h][2 * i] = bf16_lo(wq[i]) * scale_log2;
                    qr[h][2 * i + 1] = bf16_hi(wq[i]) * scale_log2;
                }
#pragma unroll
                for (int e = 0; e < C::kEPL; ++e) o[h][e] = 0.f;
                m_run[h] = -INFINITY;
                l_run[h] = 0.f;
            }
        }
        const uint8_t* Ks = ring + st * C::kStageBytes;
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
                uint32_t wk[C::kEPL / 2];
                load_bf16_words<C::kEPL>(Ks + kk * C::kRowBytes + lane * C::kEPL * 2, wk);
#pragma unroll
                for (int i2 = 0; i2 < C::kEPL / 2; ++i2) {
                    const float2 kv = make_float2(bf16_lo(wk[i2]), bf16_hi(wk[i2]));
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
            if (pass == kPasses - 1) {   // every lane is done with K (and the mask) of this stage
                __syncwarp();
                if (u + S < n) issue_k(u + S);
            }
            // the mask decides liveness: rows past S_ctx are -inf there, whatever K holds
            const float x = (mv != -INFINITY) ? part[0] + mv : -INFINITY;
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
                if (!mbar_wait_warp(&bar[2 * st + 1], ph, abort_flag)) {
                    ok = false;
                    break;
                }
            }
            // ---- O += P V for this pass's heads. Dead keys are skipped, not multiplied by
            // p = 0: their V rows (masked cache slots, rows past S_ctx) may hold anything.
#pragma unroll
            for (int kk = 0; kk < kSubKeys; ++kk) {
                if ((live_bits >> (kk * kBase)) & 1u) {
                    uint32_t wv[C::kEPL / 2];
                    load_bf16_words<C::kEPL>(Vs + kk * C::kRowBytes + lane * C::kEPL * 2, wv);
                    float pk[kHeadsPerPass];
#pragma unroll
                    for (int hh = 0; hh < kHeadsPerPass; ++hh) pk[hh] = scr[hh * kSubKeys + kk];
#pragma unroll
                    for (int i2 = 0; i2 < C::kEPL / 2; ++i2) {
                        const float2 vv = make_float2(bf16_lo(wv[i2]), bf16_hi(wv[i2]));
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
        // V of this stage is consumed: refill it with the item S ahead
        if (lane == 0 && u + S < n) issue_v(u + S);
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

// ---------------------------------------------------------------- 3. combine
// out[b,h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the partial slots of
// (b, g = h / G); a pair without live keys gives a zero row. A pair may have as
// many partials as there are warps, so the CTA splits them: kGroups groups of
// D / 4 threads (4 dims each) take slots r, r + kGroups, ..., fetch (m, l, o) of
// all of them at once and merge them with the same max-rescaling rule, and the
// groups' results are merged through shared memory.
constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
decode_combine_kernel(Workspace ws, uint16_t* __restrict__ out, int B, int Hkv, int G, int Pw) {
    constexpr int kLanesPerRow = D / 4;                       // threads that cover one o row
    constexpr int kGroups = kCombineThreads / kLanesPerRow;   // slots merged side by side
    constexpr int kBatch = 8;                                 // slots fetched together per group
    __shared__ __align__(16) float4 part_o[kGroups][kLanesPerRow];
    __shared__ float part_m[kGroups], part_l[kGroups];
    pdl_launch_dependents();  // the next call's scan may set up; it waits for this grid itself
    const int tid = threadIdx.x, lane = tid & 31;
    const int row = blockIdx.x;   // b * Hq + h
    const int Hq = Hkv * G;
    const int b = row / Hq, h = row % Hq, g = h / G, hh = h % G;
    // The scan kernel finished before this grid was launched (the stream kernel lets it
    // start only after its own wait on the scan), so the counts are final: locate the
    // partial slots while the stream kernel's last warps still run. L2 reads (.cg).
    const CountSums cs = count_sums<true>(ws.counts, B, b, lane);
    const int cb = __ldcg(ws.counts + b);
    const int r = tid / kLanesPerRow, dl = tid % kLanesPerRow, d = dl * 4;
    pdl_wait_predecessor();   // the stream kernel's partials are complete and visible
    if (cb == 0) {   // no live key: zero row (uniform branch)
        if (r == 0) *reinterpret_cast<uint2*>(out + static_cast<size_t>(row) * D + d) = make_uint2(0u, 0u);
        return;
    }
    const int T = cs.total * Hkv;
    const int c = (T + Pw - 1) / Pw;
    const int s = Hkv * cs.before + g * cb;              // first item of the pair
    const int w0 = s / c, w1 = (s + cb - 1) / c;          // warps that cover it
    const size_t slot0 = static_cast<size_t>(w0) + Hkv * cs.nz_before + g;
    const int ns = w1 - w0 + 1;

    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = r; i0 < ns; i0 += kGroups * kBatch) {
        float mb[kBatch], lb[kBatch];
        float4 ob[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {   // all loads first: one round trip per batch
            const int i = i0 + j * kGroups;
            mb[j] = -INFINITY;
            lb[j] = 0.f;
            ob[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < ns) {
                const size_t slot = slot0 + i;
                mb[j] = ws.m[slot * G + hh];
                lb[j] = ws.l[slot * G + hh];
                ob[j] = *reinterpret_cast<const float4*>(ws.o + (slot * G + hh) * D + d);
            }
        }
        float Mn = M;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) Mn = fmaxf(Mn, mb[j]);
        if (Mn == -INFINITY) continue;
        const float a = ex2_approx(M - Mn);   // 0 while M is still -inf
        L *= a;
        acc.x *= a;
        acc.y *= a;
        acc.z *= a;
        acc.w *= a;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const float wgt = ex2_approx(mb[j] - Mn);   // 0 for empty entries (m = -inf)
            L = fmaf(wgt, lb[j], L);
            acc.x = fmaf(wgt, ob[j].x, acc.x);
            acc.y = fmaf(wgt, ob[j].y, acc.y);
            acc.z = fmaf(wgt, ob[j].z, acc.z);
            acc.w = fmaf(wgt, ob[j].w, acc.w);
        }
        M = Mn;
    }
    part_o[r][dl] = acc;
    if (dl == 0) {
        part_m[r] = M;
        part_l[r] = L;
    }
    __syncthreads();
    if (r == 0) {
        float Mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < kGroups; ++j) Mt = fmaxf(Mt, part_m[j]);
        float den = 0.f;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        if (Mt != -INFINITY) {
#pragma unroll
            for (int j = 0; j < kGroups; ++j) {
                if (part_m[j] == -INFINITY) continue;
                const float wgt = ex2_approx(part_m[j] - Mt);
                const float4 oj = part_o[j][dl];
                den = fmaf(wgt, part_l[j], den);
                t.x = fmaf(wgt, oj.x, t.x);
                t.y = fmaf(wgt, oj.y, t.y);
                t.z = fmaf(wgt, oj.z, t.z);
                t.w = fmaf(wgt, oj.w, t.w);
            }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        uint2 pk;
        pk.x = pack_bf16x2(t.x * inv, t.y * inv);
        pk.y = pack_bf16x2(t.z * inv, t.w * inv);
        *reinterpret_cast<uint2*>(out + static_cast<size_t>(row) * D + d) = pk;
    }
}

}  // namespace dec
}  // namespace attn

#include "decode_mma.cuh"

namespace attn {
namespace dec {

// ---------------------------------------------------------------- host
// The stream step runs on the tensor cores (decode_mma.cuh) when num_kv_groups query heads
// share each K/V byte often enough for the CUDA-core dot products to cost issue slots that
// compete with the copies; D = 512 keeps the CUDA-core path (its O^T would not fit).
template <int D, int G>
constexpr bool use_mma() { return D <= 256 && G >= 4; }

template <int D, int G>
int launch_stream_mma(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hkv,
                      int S_ctx, float scale, const Workspace& ws, cudaStream_t stream, int* Pw) {
    using C = MmaCfg<D>;
    static std::atomic<int> ctas_for_dev[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -6;
    int P = ctas_for_dev[dev].load();
    if (P == 0) {
        if (cudaFuncSetAttribute(decode_stream_mma_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
            cudaSuccess)
            return -6;
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_stream_mma_kernel<D, G>,
                                                          C::kThreads, C::kSmemBytes) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -6;
        P = std::max(1, std::min(Cfg<D>::kMaxWarpsTotal / C::kWarps, per_sm * sms));
        ctas_for_dev[dev].store(P);
    }
    CUtensorMap tk, tv;
    const uint64_t planes = static_cast<uint64_t>(B) * Hkv;
    if (encode_map_3d_bf16(&tk, k, D, S_ctx, planes, 64, kSubKeys) ||
        encode_map_3d_bf16(&tv, v, D, S_ctx, planes, 64, kSubKeys))
        return -6;
    *Pw = P * C::kWarps;
    return launch_pdl(decode_stream_mma_kernel<D, G>, dim3(P), dim3(C::kThreads), C::kSmemBytes,
                      stream, tk, tv, q, ws, B, Hkv, S_ctx, scale * kLog2e);
}

template <int D, int G>
int launch_dg(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
              uint16_t* out, int B, int Hkv, int S_ctx, float scale, const Workspace& ws,
              cudaStream_t stream) {
    using C = Cfg<D>;
    if constexpr (use_mma<D, G>()) {
        if (launch_pdl(decode_scan_kernel, dim3(B), dim3(kScanThreads), 0, stream, mask, S_ctx, ws))
            return -6;
        int Pw = 0;
        if (launch_stream_mma<D, G>(q, k, v, B, Hkv, S_ctx, scale, ws, stream, &Pw)) return -6;
        return launch_pdl(decode_combine_kernel<D>, dim3(B * Hkv * G), dim3(kCombineThreads), 0,
                          stream, ws, out, B, Hkv, G, Pw);
    }
    static std::atomic<int> ctas_for_dev[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -6;
    int P = ctas_for_dev[dev].load();
    if (P == 0) {   // one wave: resident CTAs per SM x SMs, at most the slots the workspace holds
        if (cudaFuncSetAttribute(decode_stream_kernel<D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
            cudaSuccess)
            return -6;
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_stream_kernel<D, G>,
                                                          C::kThreads, C::kSmemBytes) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -6;
        P = std::max(1, std::min(C::kMaxWarpsTotal / C::kWarps, per_sm * sms));
        ctas_for_dev[dev].store(P);
    }
    if (launch_pdl(decode_scan_kernel, dim3(B), dim3(kScanThreads), 0, stream, mask, S_ctx, ws))
        return -6;
    if (launch_pdl(decode_stream_kernel<D, G>, dim3(P), dim3(C::kThreads), C::kSmemBytes, stream,
                   q, k, v, ws, B, Hkv, S_ctx, scale * kLog2e))
        return -6;
    return launch_pdl(decode_combine_kernel<D>, dim3(B * Hkv * G), dim3(kCombineThreads), 0, stream, ws, out,
                      B, Hkv, G, P * C::kWarps);
}

template <int D>
int launch_d(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
             uint16_t* out, int B, int Hkv, int G, int S_ctx, float scale, const Workspace& ws,
             cudaStream_t s) {
    switch (G) {
        case 1: return launch_dg<D, 1>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws, s);
        case 2: return launch_dg<D, 2>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws, s);
        case 4: return launch_dg<D, 4>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws, s);
        case 8:
            if constexpr (D <= 256) return launch_dg<D, 8>(q, k, v, mask, out, B, Hkv, S_ctx, scale, ws, s);
            return -3;   // ATTN_ERR_UNSUPPORTED: D = 512 with 8 heads per group
        default: return -3;
    }
}

// Largest problem the 32-bit item arithmetic covers: Hkv * B * ceil(S_ctx / 8) items.
inline bool items_fit(int B, int Hkv, int S_ctx) {
    return static_cast<long long>(B) * Hkv * num_sub_tiles(S_ctx) < (1ll << 30);
}

// Carves the workspace and launches scan + stream + combine on `stream`.
inline int launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* mask,
                  uint16_t* out, int B, int Hq, int Hkv, int G, int S_ctx, int D, float scale,
                  void* workspace, cudaStream_t stream) {
    const Workspace ws = carve_workspace(workspace, B, Hq, Hkv, S_ctx, D);
    switch (D) {
        case 128: return launch_d<128>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws, stream);
        case 256: return launch_d<256>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws, stream);
        case 512: return launch_d<512>(q, k, v, mask, out, B, Hkv, G, S_ctx, scale, ws, stream);
        default: return -3;
    }
}

}  // namespace dec
}  // namespace attn
