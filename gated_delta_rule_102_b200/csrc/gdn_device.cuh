// Device building blocks of the GDN decode step for sm_100a: bf16 handling, the
// per-channel causal conv with its history roll, the gate, the cluster barrier and
// the register-resident delta-rule pass over one state tile.
//
// Method: the page "spark_model/forward/qwen3_5/linear_attention.rs" (Atlas),
// steps 3 (conv + SiLU + q/k L2 norm), 4 (gate), 5 (beta), 7 (gated delta rule)
// and 8 (per-head RMSNorm) with the SiLU(z) gate of steps 9+10+11.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Bits a kernel ORs into the caller's error flag (values of the public header).
constexpr int GDN_DEVICE_ERR_SLOT_RANGE_BIT = 1;
constexpr int GDN_DEVICE_ERR_TIMEOUT_BIT = 2;
constexpr int GDN_DEVICE_ERR_SEQLEN_BIT = 4;
constexpr int GDN_DEVICE_ERR_BATCH_BIT = 8;

// The batch count of a launch: B_max, or the value a device batch count holds when
// one is given. A value outside [0, B_max] runs no sequence; `report` threads flag it.
__device__ __forceinline__ int launch_batch(const int32_t* B_dev, int B_max, int32_t* err_flag, bool report) {
    if (!B_dev) return B_max;
    const int b = *reinterpret_cast<const volatile int32_t*>(B_dev);
    if (b < 0 || b > B_max) {
        if (report && err_flag) atomicOr(err_flag, GDN_DEVICE_ERR_BATCH_BIT);
        return 0;
    }
    return b;
}

// Longest conv supported (taps) and most tokens per launch.
constexpr int kMaxConvWidth = 8;
constexpr int kMaxTokens = 16;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits) { return __uint_as_float(bits << 16); }

// float -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet).
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__device__ __forceinline__ float silu(float x) { return x / (1.0f + expf(-x)); }
__device__ __forceinline__ float sigmoid(float x) { return 1.0f / (1.0f + expf(-x)); }
// SiLU with the hardware exponential and an approximate division (relative error a
// few ulp), for the multi-token kernels' per-channel and per-output evaluations.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
// log(1 + e^x) without overflow: max(x, 0) + log1p(e^-|x|).
__device__ __forceinline__ float softplus(float x) { return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x))); }

// Step 4 and 5: decay alpha = exp(-exp(A_log) * softplus(a + dt_bias)), beta = sigmoid(b).
__device__ __forceinline__ void gate_and_beta(uint16_t a_bits, uint16_t b_bits, float A_log, float dt_bias,
                                              float& alpha, float& beta) {
    const float g = -expf(A_log) * softplus(bf16_bits_to_float(a_bits) + dt_bias);
    alpha = expf(g);
    beta = sigmoid(bf16_bits_to_float(b_bits));
}

// ---------------------------------------------------------------------------------
// Step 3 for one channel: a depthwise causal conv of width W over the slot's W-1
// stored raw inputs followed by this launch's T raw inputs, SiLU on the result.
// The window lives in registers with the newest input at the highest index, so
// every register index is a compile-time constant whatever W is. After the T tokens
// the last W-1 raw inputs are written back as the slot's history, bit for bit.
//   hist : &conv_pool[slot][0][ch], row stride C
//   x    : &qkv[seq][0][ch],        token stride C
//   w    : &conv_w[ch][0]
//   emit(t, s) receives SiLU(conv) of token t.
template <typename Emit>
__device__ __forceinline__ void conv_channel(uint16_t* hist, const uint16_t* x, const uint16_t* w,
                                             int W, int T, size_t C, Emit emit) {
    uint32_t win[kMaxConvWidth];
    float wt[kMaxConvWidth];
#pragma unroll
    for (int m = 0; m < kMaxConvWidth; ++m) {
        const int e = kMaxConvWidth - 1 - m;  // tokens before the newest history row
        const int r = W - 2 - e;              // history row held at win[m]
        win[m] = r >= 0 ? (uint32_t)hist[(size_t)r * C] : 0u;
    }
    // After the shift at token t, win[kMax-1-d] holds the input d tokens back, which
    // conv tap W-1-d multiplies.
#pragma unroll
    for (int m = 0; m < kMaxConvWidth; ++m) {
        const int d = kMaxConvWidth - 1 - m;
        wt[m] = d < W ? bf16_bits_to_float(w[W - 1 - d]) : 0.0f;
    }
    for (int t = 0; t < T; ++t) {
#pragma unroll
        for (int m = 0; m < kMaxConvWidth - 1; ++m) win[m] = win[m + 1];
        win[kMaxConvWidth - 1] = x[(size_t)t * C];
        float u = 0.0f;
#pragma unroll
        for (int m = 0; m < kMaxConvWidth; ++m) u = fmaf(wt[m], bf16_bits_to_float(win[m]), u);
        emit(t, silu(u));
    }
#pragma unroll
    for (int m = 0; m < kMaxConvWidth; ++m) {
        const int r = W - 2 - (kMaxConvWidth - 1 - m);
        if (r >= 0) hist[(size_t)r * C] = (uint16_t)win[m];
    }
}

// ---------------------------------------------------------------------------------
// Cluster barrier, split into arrive and wait so independent work can sit between.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
template <typename Tp>
__device__ __forceinline__ Tp* cluster_map(Tp* p, int rank) {
    uint64_t out;
    asm volatile("mapa.u64 %0, %1, %2;\n" : "=l"(out) : "l"((uint64_t)p), "r"(rank));
    return (Tp*)out;
}

// ---------------------------------------------------------------------------------
// Geometry of the register tile: a CTA holds S[0:DK][col0:col0+DVS] of one head.
// A thread owns RPT consecutive rows and 4 consecutive columns (one float4 per row);
// TPR threads span a row, so each row segment is read and written as whole sectors.
template <int DK, int DVS>
struct Tile {
    static constexpr int NT = (DK * DVS / 64) < 64 ? 64 : ((DK * DVS / 64) > 256 ? 256 : DK * DVS / 64);
    static constexpr int TPR = DVS / 4;
    static constexpr int RPP = NT / TPR;
    static constexpr int RPT = DK / RPP;
    static constexpr int NW = NT / 32;
    static_assert(DVS % 4 == 0 && TPR <= 32 && 32 % TPR == 0, "column slice");
    static_assert(NT % TPR == 0 && RPP <= DK && DK % RPP == 0, "row split");
};

// Shared-memory block the delta-rule pass reads: per token the raw (unnormalised)
// q and k of the k-head, the v slice and the per-token scalars.
struct TokenScalars {
    float alpha, beta;  // decay exp(g) and write strength
    float nq, nk;       // factors turning the raw q, k into the normalised (scaled) q, k
    float kq;           // k . q of the normalised vectors
};

// The gated delta rule on a register tile for tokens 0..T-1, one pass over S:
//   m = S^T k (old S), delta = beta (v - alpha m), S <- alpha S + k delta^T,
//   o = alpha S^T q + delta (k . q)   (= S_new^T q)
// qk  : [T][2*DK] raw q then raw k (shared)
// vs  : [T][DVS] v slice (shared);  os : [T][DVS] receives o (shared)
// red : [2][NW][2][DVS] scratch for the cross-warp sums (shared)
template <int DK, int DVS>
__device__ __forceinline__ void delta_rule_tile(float4 (&S)[Tile<DK, DVS>::RPT], const float* qk,
                                                const float* vs, const TokenScalars* sc, float* os,
                                                float* red, int T) {
    using Geo = Tile<DK, DVS>;
    constexpr int RPT = Geo::RPT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid % Geo::TPR, rp = tid / Geo::TPR;
    const int row0 = rp * RPT;
    for (int t = 0; t < T; ++t) {
        const float* qr = qk + t * 2 * DK;
        const float* kr = qr + DK;
        float kreg[RPT];
        float4 mk = make_float4(0.f, 0.f, 0.f, 0.f), mq = mk;
#pragma unroll
        for (int s = 0; s < RPT; ++s) {
            const float ki = kr[row0 + s], qi = qr[row0 + s];
            kreg[s] = ki;
            mk.x = fmaf(S[s].x, ki, mk.x); mk.y = fmaf(S[s].y, ki, mk.y);
            mk.z = fmaf(S[s].z, ki, mk.z); mk.w = fmaf(S[s].w, ki, mk.w);
            mq.x = fmaf(S[s].x, qi, mq.x); mq.y = fmaf(S[s].y, qi, mq.y);
            mq.z = fmaf(S[s].z, qi, mq.z); mq.w = fmaf(S[s].w, qi, mq.w);
        }
        // rows held by the other lanes of this warp with the same column group
#pragma unroll
        for (int off = Geo::TPR; off < 32; off <<= 1) {
            mk.x += __shfl_xor_sync(0xffffffffu, mk.x, off); mk.y += __shfl_xor_sync(0xffffffffu, mk.y, off);
            mk.z += __shfl_xor_sync(0xffffffffu, mk.z, off); mk.w += __shfl_xor_sync(0xffffffffu, mk.w, off);
            mq.x += __shfl_xor_sync(0xffffffffu, mq.x, off); mq.y += __shfl_xor_sync(0xffffffffu, mq.y, off);
            mq.z += __shfl_xor_sync(0xffffffffu, mq.z, off); mq.w += __shfl_xor_sync(0xffffffffu, mq.w, off);
        }
        float* rb = red + (t & 1) * (Geo::NW * 2 * DVS);
        if (lane < Geo::TPR) {
            reinterpret_cast<float4*>(rb + (warp * 2 + 0) * DVS)[cg] = mk;
            reinterpret_cast<float4*>(rb + (warp * 2 + 1) * DVS)[cg] = mq;
        }
        __syncthreads();
        mk = make_float4(0.f, 0.f, 0.f, 0.f);
        mq = mk;
#pragma unroll
        for (int w = 0; w < Geo::NW; ++w) {
            const float4 a = reinterpret_cast<const float4*>(rb + (w * 2 + 0) * DVS)[cg];
            const float4 b = reinterpret_cast<const float4*>(rb + (w * 2 + 1) * DVS)[cg];
            mk.x += a.x; mk.y += a.y; mk.z += a.z; mk.w += a.w;
            mq.x += b.x; mq.y += b.y; mq.z += b.z; mq.w += b.w;
        }
        const TokenScalars c = sc[t];
        const float4 v = reinterpret_cast<const float4*>(vs + t * DVS)[cg];
        const float am = c.alpha * c.nk, aq = c.alpha * c.nq;
        float4 d, o;
        d.x = c.beta * fmaf(-am, mk.x, v.x); d.y = c.beta * fmaf(-am, mk.y, v.y);
        d.z = c.beta * fmaf(-am, mk.z, v.z); d.w = c.beta * fmaf(-am, mk.w, v.w);
        o.x = fmaf(aq, mq.x, d.x * c.kq); o.y = fmaf(aq, mq.y, d.y * c.kq);
        o.z = fmaf(aq, mq.z, d.z * c.kq); o.w = fmaf(aq, mq.w, d.w * c.kq);
        if (rp == 0) reinterpret_cast<float4*>(os + t * DVS)[cg] = o;
        // the raw k times nk is the normalised k: fold nk into delta
        const float4 dn = make_float4(d.x * c.nk, d.y * c.nk, d.z * c.nk, d.w * c.nk);
#pragma unroll
        for (int s = 0; s < RPT; ++s) {
            S[s].x = fmaf(c.alpha, S[s].x, kreg[s] * dn.x); S[s].y = fmaf(c.alpha, S[s].y, kreg[s] * dn.y);
            S[s].z = fmaf(c.alpha, S[s].z, kreg[s] * dn.z); S[s].w = fmaf(c.alpha, S[s].w, kreg[s] * dn.w);
        }
    }
}

// Per-token sums over the raw q and k of one k-head held in shared memory:
// |q|^2, |k|^2 and q.k, one warp per token. Writes nq, nk, kq of `sc`.
template <int DK>
__device__ __forceinline__ void qk_norms(const float* qk, TokenScalars* sc, int T, float l2_eps, float q_scale,
                                         int nwarps) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = warp; t < T; t += nwarps) {
        const float* qr = qk + t * 2 * DK;
        const float* kr = qr + DK;
        float sq = 0.f, sk = 0.f, dot = 0.f;
        for (int i = lane; i < DK; i += 32) {
            const float a = qr[i], b = kr[i];
            sq = fmaf(a, a, sq);
            sk = fmaf(b, b, sk);
            dot = fmaf(a, b, dot);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            dot += __shfl_xor_sync(0xffffffffu, dot, off);
        }
        if (lane == 0) {
            const float nq = rsqrtf(sq + l2_eps) * q_scale, nk = rsqrtf(sk + l2_eps);
            sc[t].nq = nq;
            sc[t].nk = nk;
            sc[t].kq = dot * nq * nk;
        }
    }
}

}  // namespace gdn

namespace gdn {

// ---------------------------------------------------------------------------------
// TMA bulk copies (global -> shared, completion counted on an mbarrier) and bounded
// mbarrier waits. No multicast anywhere.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// Makes the initialised barrier visible to the async proxy and the cluster.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Like mbar_try_wait, suspending for at most about `hint_ns` while the phase is open.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
// Bound on every wait inside the kernels, in cycles of the SM's own clock (a second at
// 2 GHz, longer at lower clocks). The SM cycle counter only moves forward while the
// warp waits; the global timer is not used for this, since it may be adjusted while a
// kernel runs and a jump would end a healthy wait (an unsigned difference across a
// backward step reads as an enormous elapsed time).
constexpr uint64_t kWaitTimeoutCycles = 2000000000ull;
// Waits for phase `parity` of the barrier; gives up after about `timeout_cycles` SM
// cycles and returns false. `give_up` is polled now and then so a CTA can stop waiting
// early.
// Suspend-time hint of each poll, in nanoseconds (0: polls without a hint). A build-time
// tuning constant.
#ifndef GDN_WAIT_HINT_NS
#define GDN_WAIT_HINT_NS 1000
#endif
__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity) {
    if (GDN_WAIT_HINT_NS > 0) return mbar_try_wait_hint(bar, parity, GDN_WAIT_HINT_NS);
    return mbar_try_wait(bar, parity);
}
template <typename GiveUp>
__device__ __forceinline__ bool mbar_wait_deadline(uint64_t* bar, uint32_t parity, uint64_t timeout_cycles,
                                                   GiveUp give_up) {
    if (mbar_poll(bar, parity)) return true;
    const uint64_t t0 = clock64();
    for (uint32_t i = 1;; ++i) {
        if (mbar_poll(bar, parity)) return true;
        if ((i & 15) == 0) {
            if (give_up()) return false;
            if ((uint64_t)clock64() - t0 > timeout_cycles) return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t timeout_cycles = kWaitTimeoutCycles) {
    return mbar_wait_deadline(bar, parity, timeout_cycles, [] { return false; });
}
// One bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) into
// this CTA's shared memory, counted on `bar`.
__device__ __forceinline__ void tma_load_1d(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), and the arrival
// on `bar` once all of this thread's earlier such copies have landed (the arrival
// counts toward the barrier's expected count: it does not add to it).
__device__ __forceinline__ void cp_async_16(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}

// Bulk prefetch of global memory into L2 (a hint: no completion, no ordering).
// src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src_gmem, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src_gmem), "r"(bytes) : "memory");
}

// The gated delta rule on a DK x DVS tile held in shared memory, for tokens 0..T-1.
// Same arithmetic as delta_rule_tile; S lives in shared memory between tokens and
// each thread reads it twice per token (reductions, then update), so registers stay
// few. After the last token the updated rows go straight to global memory `Sg`
// (this thread's first float4, row pitch `pitch4` float4s) with streaming stores.
template <int DK, int DVS>
__device__ __forceinline__ void delta_rule_smem(float* tile, const float* qk, const float* vs, const TokenScalars* sc,
                                                float* os, float* red, int T, float4* Sg, size_t pitch4) {
    using Geo = Tile<DK, DVS>;
    constexpr int RPT = Geo::RPT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid % Geo::TPR, rp = tid / Geo::TPR;
    const int row0 = rp * RPT;
    float4* tl = reinterpret_cast<float4*>(tile) + (size_t)row0 * (DVS / 4) + cg;
    for (int t = 0; t < T; ++t) {
        const float* qr = qk + t * 2 * DK;
        const float* kr = qr + DK;
        float4 mk = make_float4(0.f, 0.f, 0.f, 0.f), mq = mk;
#pragma unroll
        for (int s = 0; s < RPT; ++s) {
            const float4 v = tl[s * (DVS / 4)];
            const float ki = kr[row0 + s], qi = qr[row0 + s];
            mk.x = fmaf(v.x, ki, mk.x); mk.y = fmaf(v.y, ki, mk.y);
            mk.z = fmaf(v.z, ki, mk.z); mk.w = fmaf(v.w, ki, mk.w);
            mq.x = fmaf(v.x, qi, mq.x); mq.y = fmaf(v.y, qi, mq.y);
            mq.z = fmaf(v.z, qi, mq.z); mq.w = fmaf(v.w, qi, mq.w);
        }
#pragma unroll
        for (int off = Geo::TPR; off < 32; off <<= 1) {
            mk.x += __shfl_xor_sync(0xffffffffu, mk.x, off); mk.y += __shfl_xor_sync(0xffffffffu, mk.y, off);
            mk.z += __shfl_xor_sync(0xffffffffu, mk.z, off); mk.w += __shfl_xor_sync(0xffffffffu, mk.w, off);
            mq.x += __shfl_xor_sync(0xffffffffu, mq.x, off); mq.y += __shfl_xor_sync(0xffffffffu, mq.y, off);
            mq.z += __shfl_xor_sync(0xffffffffu, mq.z, off); mq.w += __shfl_xor_sync(0xffffffffu, mq.w, off);
        }
        float* rb = red + (t & 1) * (Geo::NW * 2 * DVS);
        if (lane < Geo::TPR) {
            reinterpret_cast<float4*>(rb + (warp * 2 + 0) * DVS)[cg] = mk;
            reinterpret_cast<float4*>(rb + (warp * 2 + 1) * DVS)[cg] = mq;
        }
        __syncthreads();
        mk = make_float4(0.f, 0.f, 0.f, 0.f);
        mq = mk;
#pragma unroll
        for (int w = 0; w < Geo::NW; ++w) {
            const float4 a = reinterpret_cast<const float4*>(rb + (w * 2 + 0) * DVS)[cg];
            const float4 b = reinterpret_cast<const float4*>(rb + (w * 2 + 1) * DVS)[cg];
            mk.x += a.x; mk.y += a.y; mk.z += a.z; mk.w += a.w;
            mq.x += b.x; mq.y += b.y; mq.z += b.z; mq.w += b.w;
        }
        const TokenScalars c = sc[t];
        const float4 v = reinterpret_cast<const float4*>(vs + t * DVS)[cg];
        const float am = c.alpha * c.nk, aq = c.alpha * c.nq;
        float4 d, o;
        d.x = c.beta * fmaf(-am, mk.x, v.x); d.y = c.beta * fmaf(-am, mk.y, v.y);
        d.z = c.beta * fmaf(-am, mk.z, v.z); d.w = c.beta * fmaf(-am, mk.w, v.w);
        o.x = fmaf(aq, mq.x, d.x * c.kq); o.y = fmaf(aq, mq.y, d.y * c.kq);
        o.z = fmaf(aq, mq.z, d.z * c.kq); o.w = fmaf(aq, mq.w, d.w * c.kq);
        if (rp == 0) reinterpret_cast<float4*>(os + t * DVS)[cg] = o;
        const float4 dn = make_float4(d.x * c.nk, d.y * c.nk, d.z * c.nk, d.w * c.nk);
        const bool last = t == T - 1;
#pragma unroll
        for (int s = 0; s < RPT; ++s) {
            float4 w = tl[s * (DVS / 4)];
            const float ki = kr[row0 + s];
            w.x = fmaf(c.alpha, w.x, ki * dn.x); w.y = fmaf(c.alpha, w.y, ki * dn.y);
            w.z = fmaf(c.alpha, w.z, ki * dn.z); w.w = fmaf(c.alpha, w.w, ki * dn.w);
            if (last) __stcs(Sg + (size_t)s * pitch4, w);
            else tl[s * (DVS / 4)] = w;
        }
    }
}

}  // namespace gdn

namespace gdn {

// ---------------------------------------------------------------------------------
// Distributed-shared-memory messages completed on the receiver's mbarrier, and the
// async-proxy fence used before a bulk copy reuses a buffer the threads have read.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ uint32_t cluster_map_u32(uint32_t smem_cta_addr, int rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(out) : "r"(smem_cta_addr), "r"(rank));
    return out;
}
// Store one float into the shared memory of the cluster CTA that owns `remote_addr`
// and count 4 bytes on that CTA's mbarrier `remote_bar` (both shared::cluster).
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];\n" ::"r"(remote_addr),
                 "r"(__float_as_uint(v)), "r"(remote_bar)
                 : "memory");
}
// Named barrier over `threads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}
// Named barrier that also returns whether `pred` held in every participating thread:
// warps sharing later named barriers leave a loop together or not at all.
__device__ __forceinline__ bool named_barrier_and(int id, int threads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

}  // namespace gdn

namespace gdn {
// Two floats into another cluster CTA's shared memory (8-byte aligned), counted as
// 8 bytes on that CTA's mbarrier.
__device__ __forceinline__ void st_async_f32x2(uint32_t remote_addr, float a, float b, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];\n" ::"r"(
                     remote_addr),
                 "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(remote_bar)
                 : "memory");
}
}  // namespace gdn
