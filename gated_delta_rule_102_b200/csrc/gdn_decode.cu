// The fused GDN decode step: conv update, gate, gated delta rule and gated RMSNorm
// in one launch (steps 3 to 8 and the SiLU(z) gate of steps 9+10+11 on the page
// "spark_model/forward/qwen3_5/linear_attention.rs").
//
// This file holds the launcher that picks the kernel for a launch, and the kernel
// for single-token launches over few sequences:
//  * one token, enough (sequence, k-head) groups to fill the GPU twice: the
//    persistent pipelined kernel (gdn_decode_persistent.cu);
//  * several tokens: the multi-token kernel (gdn_decode_mt.cu);
//  * otherwise the cluster kernel below.
//
// Cluster kernel. One thread-block cluster per (sequence, k-head). Its G*NS CTAs
// are the G v-heads that share the k-head (v-head h reads k-head h / G) times NS
// column slices of dv. CTA (v-head h, slice sl) owns state columns
// [sl*DVS, (sl+1)*DVS) of head h: it stages that DK x DVS fp32 tile from HBM into
// shared memory by TMA, runs the token on it, and writes it back in place. The
// columns of S are independent under the update (column j needs only S[:, j], k, q
// and v_j), so the slices never exchange state.
//
// Conv ownership. Every channel's conv history is read and rolled by exactly one CTA
// of the grid: the CTA's own v columns, plus a 1/(G*NS) share of its k-head's q and k
// channels. The q/k shares are pushed into every cluster CTA's shared memory
// (distributed shared memory, plain stores) so each CTA sees the whole raw q and k.
// The per-head RMSNorm sums of the NS slices of a v-head travel the same way.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kMaxCluster = 8;
// Launches with at most this many tokens stage the state tile in shared memory
// (bandwidth-bound); longer ones run the multi-token kernel, which keeps it in
// registers across tokens (ALU-bound).
#ifndef GDN_MAX_TOKENS_STAGED
#define GDN_MAX_TOKENS_STAGED 1
#endif
constexpr int kMaxTokensStaged = GDN_MAX_TOKENS_STAGED;
// Single-token launches with at least this many (sequence, k-head) groups per
// co-resident cluster run the persistent kernel.
#ifndef GDN_PERSISTENT_MIN_WAVES
#define GDN_PERSISTENT_MIN_WAVES 2
#endif
constexpr int kPersistentMinWaves = GDN_PERSISTENT_MIN_WAVES;

template <int DK, int DVS>
struct FusedSmem {
    using Geo = Tile<DK, DVS>;
    // float offsets; every block starts on a 16-byte boundary
    static __host__ __device__ constexpr int round4(int n) { return (n + 3) & ~3; }
    static __host__ __device__ int qk(int) { return 0; }
    static __host__ __device__ int vs(int T) { return qk(T) + round4(T * 2 * DK); }
    static __host__ __device__ int os(int T) { return vs(T) + round4(T * DVS); }
    static __host__ __device__ int red(int T) { return os(T) + round4(T * DVS); }
    static __host__ __device__ int sc(int T) { return red(T) + 2 * Geo::NW * 2 * DVS; }
    static __host__ __device__ int part(int T) { return sc(T) + round4(T * (int)(sizeof(TokenScalars) / 4)); }
    static __host__ __device__ int total_floats(int T, int NS) { return part(T) + round4(T * NS); }
};

template <int DK, int DVS>
struct TmaSmem {
    using F = FusedSmem<DK, DVS>;
    static __host__ __device__ int tile() { return 0; }
    static __host__ __device__ int rest(int) { return DK * DVS; }  // FusedSmem blocks follow the tile
    static __host__ __device__ size_t bar_bytes_offset(int T, int NS) {
        return ((size_t)(DK * DVS + F::total_floats(T, NS)) * 4 + 7) & ~(size_t)7;
    }
    static __host__ __device__ size_t total_bytes(int T, int NS) { return bar_bytes_offset(T, NS) + 8; }
};

// The cluster kernel (work decomposition at the top of this file). The state tile is
// staged into shared memory before the conv work: by TMA bulk copies when the slice is
// whole rows, else by 16-byte cp.async from every thread, completing on one mbarrier.
// The copies run beside the conv and the cluster barriers, and the tile occupies no
// registers; the update streams back to HBM from registers.
template <int DK, int DVS>
__global__ void __launch_bounds__(Tile<DK, DVS>::NT)
decode_fused_tma_kernel(const DecodeArgs p) {
    using Geo = Tile<DK, DVS>;
    using L = FusedSmem<DK, DVS>;
    constexpr int NT = Geo::NT;
    extern __shared__ __align__(128) float4 smem4[];
    float* tile = reinterpret_cast<float*>(smem4);
    float* smem = tile + DK * DVS;
    uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(smem4) +
                                                TmaSmem<DK, DVS>::bar_bytes_offset(p.T, p.NS));

    const int T = p.T, G = p.sh.Hv / p.sh.Hk, NS = p.NS, CS = G * NS;
    const int dv = p.sh.dv, C = p.sh.C;
    const int cid = blockIdx.x / CS, rank = blockIdx.x - cid * CS;
    const int seq = cid / p.sh.Hk, hk = cid - seq * p.sh.Hk;
    const int gi = rank / NS, sl = rank - gi * NS;
    const int h = hk * G + gi, col0 = sl * DVS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) {
        // a contiguous tile comes by bulk copies (one arrival with the bytes); a strided
        // one by 16-byte asynchronous copies from every thread (one arrival each)
        mbar_init(bar, DVS == dv ? 1 : NT);
        mbar_init_fence();
    }
    __syncthreads();
    if (CS > 1) cluster_arrive_relaxed();  // B0
    // With programmatic dependent launch this grid may start while the previous one
    // drains: nothing is read before that grid has completed.
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    // a sequence past the launch's batch count: the whole cluster leaves (seq is the cluster's)
    if (seq >= launch_batch(p.B_dev, p.B, p.err_flag, blockIdx.x == 0 && tid == 0)) return;
    const int slot = __ldg(p.slots + seq);
    if (slot < 0 || slot >= p.P) {
        if (tid == 0 && rank == 0 && p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        return;
    }
    const float* Sbase = p.state_pool + ((size_t)slot * p.sh.Hv + h) * (size_t)DK * dv + col0;
    // ---- stage the DK x DVS state tile in
    if (DVS == dv) {  // contiguous tile: bulk copies of DK/32 rows each
        if (warp == 0) {
            if (lane == 0) mbar_arrive_expect_tx(bar, DK * DVS * 4);
            __syncwarp();
            constexpr int rows = DK >= 32 ? DK / 32 : 1;
            for (int r = lane * rows; r < DK; r += 32 * rows)
                tma_load_1d(tile + (size_t)r * DVS, Sbase + (size_t)r * dv, rows * DVS * 4, bar);
        }
    } else {  // rows of DVS columns at the pool's row stride: 16-byte copies from every thread
        constexpr int VPR = DVS / 4;
        for (int i = tid; i < DK * VPR; i += NT) {
            const int r = i / VPR, c = (i - r * VPR) * 4;
            cp_async_16(tile + (size_t)r * DVS + c, Sbase + (size_t)r * dv + c);
        }
        cp_async_arrive(bar);
    }

    float* qk = smem + L::qk(T);
    float* vs = smem + L::vs(T);
    float* os = smem + L::os(T);
    float* red = smem + L::red(T);
    TokenScalars* sc = reinterpret_cast<TokenScalars*>(smem + L::sc(T));
    float* part = smem + L::part(T);

    if (tid < T) {
        const size_t i = ((size_t)seq * T + tid) * p.sh.Hv + h;
        gate_and_beta(p.a[i], p.b[i], p.A_log[h], p.dt_bias[h], sc[tid].alpha, sc[tid].beta);
    }
    if (CS > 1) cluster_wait_acquire();
    const int qk_lo = (rank * 2 * DK) / CS, qk_hi = ((rank + 1) * 2 * DK) / CS;
    const int nqk = qk_hi - qk_lo;
    uint16_t* hist_base = p.conv_pool + (size_t)slot * (p.sh.W - 1) * C;
    const uint16_t* x_base = p.qkv + (size_t)seq * T * C;
    for (int c = tid; c < nqk + DVS; c += NT) {
        if (c < nqk) {
            const int j = qk_lo + c;
            const int ch = j < DK ? hk * DK + j : p.sh.Hk * DK + hk * DK + (j - DK);
            conv_channel(hist_base + ch, x_base + ch, p.conv_w + (size_t)ch * p.sh.W, p.sh.W, T, (size_t)C,
                         [&](int t, float s) {
                             float* dst = qk + t * 2 * DK + j;
                             if (CS > 1) {
                                 for (int r = 0; r < CS; ++r) *cluster_map(dst, r) = s;
                             } else {
                                 *dst = s;
                             }
                         });
        } else {
            const int jj = c - nqk;
            const int ch = 2 * p.sh.Hk * DK + h * dv + col0 + jj;
            conv_channel(hist_base + ch, x_base + ch, p.conv_w + (size_t)ch * p.sh.W, p.sh.W, T, (size_t)C,
                         [&](int t, float s) { vs[t * DVS + jj] = s; });
        }
    }
    if (CS > 1) {  // B1
        cluster_arrive_release();
        cluster_wait_acquire();
    } else {
        __syncthreads();
    }
    qk_norms<DK>(qk, sc, T, p.sh.l2_eps, p.sh.q_scale, Geo::NW);
    const bool ready = mbar_wait_bounded(bar, 0);
    const bool timed_out = __syncthreads_or(!ready);
    if (!timed_out) {
        const int cg = tid % Geo::TPR, rp = tid / Geo::TPR;
        float4* Sg = reinterpret_cast<float4*>(const_cast<float*>(Sbase)) + (size_t)(rp * Geo::RPT) * (dv / 4) + cg;
        delta_rule_smem<DK, DVS>(tile, qk, vs, sc, os, red, T, Sg, dv / 4);
    } else if (tid == 0 && p.err_flag) {
        atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
    }
    __syncthreads();
    for (int t = warp; t < T; t += Geo::NW) {
        float acc = 0.f;
        for (int j = lane; j < DVS; j += 32) acc = fmaf(os[t * DVS + j], os[t * DVS + j], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            float* dst = part + t * NS + sl;
            if (NS > 1) {
                for (int u = 0; u < NS; ++u) *cluster_map(dst, gi * NS + u) = acc;
            } else {
                *dst = acc;
            }
        }
    }
    if (CS > 1 && NS > 1) {  // B2
        cluster_arrive_release();
        cluster_wait_acquire();
    } else {
        __syncthreads();
    }
    if (timed_out) {  // the tile never arrived: wait (bounded) for the copies, write nothing
        mbar_wait_bounded(bar, 0);
        return;
    }
    const float inv_dv = 1.0f / (float)dv;
    for (int idx = tid; idx < T * DVS; idx += NT) {
        const int t = idx / DVS, j = idx - t * DVS;
        float ss = 0.f;
        for (int u = 0; u < NS; ++u) ss += part[t * NS + u];
        const float inv = rsqrtf(ss * inv_dv + p.sh.rms_eps);
        const size_t o_i = (((size_t)seq * T + t) * p.sh.Hv + h) * dv + col0 + j;
        const float y = os[t * DVS + j] * inv * bf16_bits_to_float(p.norm_w[col0 + j]) *
                        silu(bf16_bits_to_float(p.z[o_i]));
        p.out[o_i] = float_to_bf16_bits(y);
        if (p.out_f32) p.out_f32[o_i] = y;
    }
}

template <int DK, int DVS>
cudaError_t launch_tma(const DecodeArgs& a, cudaStream_t stream) {
    using Geo = Tile<DK, DVS>;
    const int G = a.sh.Hv / a.sh.Hk, CS = G * a.NS;
    const size_t smem = TmaSmem<DK, DVS>::total_bytes(a.T, a.NS);
    auto kern = decode_fused_tma_kernel<DK, DVS>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.sh.Hk * CS));
    cfg.blockDim = dim3(Geo::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int DK>
cudaError_t dispatch_dvs(const DecodeArgs& a, int dvs, cudaStream_t stream) {
    switch (dvs) {
        case 16: return launch_tma<DK, 16>(a, stream);
        case 32: return launch_tma<DK, 32>(a, stream);
        case 64: return launch_tma<DK, 64>(a, stream);
        case 128: return launch_tma<DK, 128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

int decode_column_splits(int B, int Hv, int G, int dv) {
#ifdef GDN_DECODE_SPLITS_OVERRIDE
    {  // build-time tuning override, used only when the shape allows it
        const int ns = GDN_DECODE_SPLITS_OVERRIDE;
        if (G * ns <= kMaxCluster && dv % ns == 0 && dv / ns >= 16) return ns;
    }
#endif
    // Split the v columns while the cluster fits and the slice keeps >= 64 columns;
    // small batches split further (down to 16 columns) so the grid covers the GPU.
    int ns = 1;
    while (G * ns * 2 <= kMaxCluster && dv / (ns * 2) >= 64) ns *= 2;
    while (G * ns * 2 <= kMaxCluster && dv / (ns * 2) >= 16 && (long)B * Hv * ns < 2 * 148) ns *= 2;
    return ns;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t stream) {
    if (persistent_supported(a)) {  // single token, many groups: the persistent pipelined kernel
        int cap = 0;
        cudaError_t e = persistent_capacity(a, &cap);
        if (e != cudaSuccess) return e;
        if (cap > 0 && (long)a.B * a.sh.Hk >= (long)kPersistentMinWaves * cap) return launch_decode_persistent(a, stream);
    }
    if (a.T > kMaxTokensStaged) {  // several tokens: the state stays in registers across them
        if (!multitoken_supported(a)) return cudaErrorInvalidValue;
        return launch_decode_multitoken(a, stream);
    }
    const int dvs = a.sh.dv / a.NS;
    switch (a.sh.dk) {
        case 16: return dispatch_dvs<16>(a, dvs, stream);
        case 32: return dispatch_dvs<32>(a, dvs, stream);
        case 64: return dispatch_dvs<64>(a, dvs, stream);
        case 128: return dispatch_dvs<128>(a, dvs, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gdn
