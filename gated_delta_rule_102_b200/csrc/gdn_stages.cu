// The three stages of the GDN decode step as separate launches, for bisection and
// for callers that want the intermediates (the page's step-by-step dispatch on
// "spark_model/forward/qwen3_5/linear_attention.rs": step 3 conv, steps 4, 5, 7
// recurrence, step 8 + SiLU(z) gate). They share the device building blocks of the
// fused kernel, so a parity failure of the fused path can be pinned to one stage.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 128;

// One CTA per (sequence, head block): blocks 0..Hk-1 are the Q heads, Hk..2Hk-1 the
// K heads, then the Hv V heads. Each thread convolves one channel for all T tokens.
__global__ void __launch_bounds__(kConvThreads) conv_update_kernel(const ConvArgs p) {
    extern __shared__ float buf[];  // [T][width] SiLU outputs, then per-token norms
    const int nseg = 2 * p.sh.Hk + p.sh.Hv;
    const int seq = blockIdx.x / nseg, seg = blockIdx.x - seq * nseg;
    const int T = p.T, C = p.sh.C, dk = p.sh.dk, dv = p.sh.dv;
    const int slot = __ldg(p.slots + seq);
    if (slot < 0 || slot >= p.P) {
        if (threadIdx.x == 0 && seg == 0 && p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        return;
    }
    const bool is_v = seg >= 2 * p.sh.Hk;
    const int width = is_v ? dv : dk;
    const int ch0 = is_v ? 2 * p.sh.Hk * dk + (seg - 2 * p.sh.Hk) * dv : seg * dk;
    uint16_t* hist = p.conv_pool + (size_t)slot * (p.sh.W - 1) * C;
    const uint16_t* x = p.qkv + (size_t)seq * T * C;
    for (int c = threadIdx.x; c < width; c += kConvThreads) {
        const int ch = ch0 + c;
        conv_channel(hist + ch, x + ch, p.conv_w + (size_t)ch * p.sh.W, p.sh.W, T, (size_t)C,
                     [&](int t, float s) { buf[t * width + c] = s; });
    }
    __syncthreads();
    if (is_v) {
        const int h = seg - 2 * p.sh.Hk;
        for (int i = threadIdx.x; i < T * dv; i += kConvThreads) {
            const int t = i / dv, j = i - t * dv;
            p.v[(((size_t)seq * T + t) * p.sh.Hv + h) * dv + j] = buf[i];
        }
        return;
    }
    // L2 norm per token over the head's dk channels, eps inside the root; q also scaled
    float* scale = buf + T * width;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool is_q = seg < p.sh.Hk;
    for (int t = warp; t < T; t += kConvThreads / 32) {
        float ss = 0.f;
        for (int i = lane; i < dk; i += 32) ss = fmaf(buf[t * dk + i], buf[t * dk + i], ss);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (lane == 0) scale[t] = rsqrtf(ss + p.sh.l2_eps) * (is_q ? p.sh.q_scale : 1.0f);
    }
    __syncthreads();
    const int head = is_q ? seg : seg - p.sh.Hk;
    float* dst = is_q ? p.q : p.k;
    for (int i = threadIdx.x; i < T * dk; i += kConvThreads) {
        const int t = i / dk, j = i - t * dk;
        dst[(((size_t)seq * T + t) * p.sh.Hk + head) * dk + j] = buf[i] * scale[t];
    }
}

template <int DK, int DVS>
struct RecSmem {
    using Geo = Tile<DK, DVS>;
    static __host__ __device__ constexpr int round4(int n) { return (n + 3) & ~3; }
    static __host__ __device__ int qk(int) { return 0; }
    static __host__ __device__ int vs(int T) { return round4(T * 2 * DK); }
    static __host__ __device__ int os(int T) { return vs(T) + round4(T * DVS); }
    static __host__ __device__ int red(int T) { return os(T) + round4(T * DVS); }
    static __host__ __device__ int sc(int T) { return red(T) + 2 * Geo::NW * 2 * DVS; }
    static __host__ __device__ int total_floats(int T) { return sc(T) + round4(T * (int)(sizeof(TokenScalars) / 4)); }
};

// One CTA per (sequence, v-head, column slice); q, k already normalised.
template <int DK, int DVS>
__global__ void __launch_bounds__(Tile<DK, DVS>::NT) recurrent_kernel(const RecurrentArgs p) {
    using Geo = Tile<DK, DVS>;
    using L = RecSmem<DK, DVS>;
    constexpr int RPT = Geo::RPT, NT = Geo::NT;
    extern __shared__ float4 smem4[];
    float* smem = reinterpret_cast<float*>(smem4);
    const int T = p.T, NS = p.NS, dv = p.sh.dv, Hv = p.sh.Hv, Hk = p.sh.Hk;
    const int unit = blockIdx.x / NS, sl = blockIdx.x - unit * NS;
    const int seq = unit / Hv, h = unit - seq * Hv, hk = h / (Hv / Hk), col0 = sl * DVS;
    const int tid = threadIdx.x;
    const int slot = __ldg(p.slots + seq);
    if (slot < 0 || slot >= p.P) {
        if (tid == 0 && h == 0 && sl == 0 && p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        return;
    }
    float4 S[RPT];
    const int cg = tid % Geo::TPR, rp = tid / Geo::TPR;
    float4* Sg = reinterpret_cast<float4*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)DK * dv + col0) +
                 (size_t)(rp * RPT) * (dv / 4) + cg;
#pragma unroll
    for (int s = 0; s < RPT; ++s) S[s] = __ldcs(Sg + (size_t)s * (dv / 4));

    float* qk = smem + L::qk(T);
    float* vs = smem + L::vs(T);
    float* os = smem + L::os(T);
    float* red = smem + L::red(T);
    TokenScalars* sc = reinterpret_cast<TokenScalars*>(smem + L::sc(T));
    for (int i = tid; i < T * 2 * DK; i += NT) {
        const int t = i / (2 * DK), j = i - t * 2 * DK;
        const float* src = j < DK ? p.q : p.k;
        qk[i] = src[(((size_t)seq * T + t) * Hk + hk) * DK + (j < DK ? j : j - DK)];
    }
    for (int i = tid; i < T * DVS; i += NT) {
        const int t = i / DVS, j = i - t * DVS;
        vs[i] = p.v[(((size_t)seq * T + t) * Hv + h) * dv + col0 + j];
    }
    if (tid < T) {
        const size_t i = ((size_t)seq * T + tid) * Hv + h;
        gate_and_beta(p.a[i], p.b[i], p.A_log[h], p.dt_bias[h], sc[tid].alpha, sc[tid].beta);
    }
    __syncthreads();
    {  // k . q per token (inputs are already normalised: unit factors)
        const int lane = tid & 31, warp = tid >> 5;
        for (int t = warp; t < T; t += Geo::NW) {
            float dot = 0.f;
            for (int i = lane; i < DK; i += 32) dot = fmaf(qk[t * 2 * DK + i], qk[t * 2 * DK + DK + i], dot);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            if (lane == 0) {
                sc[t].nq = 1.0f;
                sc[t].nk = 1.0f;
                sc[t].kq = dot;
            }
        }
    }
    __syncthreads();
    delta_rule_tile<DK, DVS>(S, qk, vs, sc, os, red, T);
#pragma unroll
    for (int s = 0; s < RPT; ++s) __stcs(Sg + (size_t)s * (dv / 4), S[s]);
    __syncthreads();
    for (int i = tid; i < T * DVS; i += NT) {
        const int t = i / DVS, j = i - t * DVS;
        p.o[(((size_t)seq * T + t) * Hv + h) * dv + col0 + j] = os[i];
    }
}

template <int DK, int DVS>
cudaError_t launch_rec_tile(const RecurrentArgs& a, cudaStream_t stream) {
    const size_t smem = (size_t)RecSmem<DK, DVS>::total_floats(a.T) * sizeof(float);
    auto kern = recurrent_kernel<DK, DVS>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<dim3((unsigned)(a.B * a.sh.Hv * a.NS)), dim3(Tile<DK, DVS>::NT), smem, stream>>>(a);
    return cudaGetLastError();
}

template <int DK>
cudaError_t rec_dispatch_dvs(const RecurrentArgs& a, int dvs, cudaStream_t stream) {
    switch (dvs) {
        case 16: return launch_rec_tile<DK, 16>(a, stream);
        case 32: return launch_rec_tile<DK, 32>(a, stream);
        case 64: return launch_rec_tile<DK, 64>(a, stream);
        case 128: return launch_rec_tile<DK, 128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

constexpr int kNormThreads = 128;

// One warp per (sequence, token, v-head) row of dv values.
__global__ void __launch_bounds__(kNormThreads) gated_rmsnorm_kernel(const NormArgs p) {
    const int warps = kNormThreads / 32;
    const int row = blockIdx.x * warps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= p.rows) return;
    const int dv = p.sh.dv;
    const float* o = p.o + (size_t)row * dv;
    float ss = 0.f;
    for (int j = lane; j < dv; j += 32) ss = fmaf(o[j], o[j], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss / (float)dv + p.sh.rms_eps);
    for (int j = lane; j < dv; j += 32) {
        const size_t i = (size_t)row * dv + j;
        const float y = o[j] * inv * bf16_bits_to_float(p.norm_w[j]) * silu(bf16_bits_to_float(p.z[i]));
        p.out[i] = float_to_bf16_bits(y);
        if (p.out_f32) p.out_f32[i] = y;
    }
}

}  // namespace

int recurrent_column_splits(int B, int Hv, int dv) {
    int ns = 1;
    while (dv / (ns * 2) >= 64) ns *= 2;
    while (dv / (ns * 2) >= 16 && (long)B * Hv * ns < 2 * 148) ns *= 2;
    return ns;
}

cudaError_t launch_conv_update(const ConvArgs& a, cudaStream_t stream) {
    const int width = a.sh.dk > a.sh.dv ? a.sh.dk : a.sh.dv;
    const size_t smem = (size_t)(a.T * width + a.T) * sizeof(float);
    conv_update_kernel<<<dim3((unsigned)(a.B * (2 * a.sh.Hk + a.sh.Hv))), dim3(kConvThreads), smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_recurrent(const RecurrentArgs& a, cudaStream_t stream) {
    const int dvs = a.sh.dv / a.NS;
    switch (a.sh.dk) {
        case 16: return rec_dispatch_dvs<16>(a, dvs, stream);
        case 32: return rec_dispatch_dvs<32>(a, dvs, stream);
        case 64: return rec_dispatch_dvs<64>(a, dvs, stream);
        case 128: return rec_dispatch_dvs<128>(a, dvs, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_gated_rmsnorm(const NormArgs& a, cudaStream_t stream) {
    const int warps = kNormThreads / 32;
    gated_rmsnorm_kernel<<<dim3((unsigned)((a.rows + warps - 1) / warps)), dim3(kNormThreads), 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace gdn
