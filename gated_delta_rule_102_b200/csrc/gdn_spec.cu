// Commit of a speculative verify: each sequence keeps the state and conv history
// after the first n_accept[b] of its drafted tokens.
//
// The verify call (the multi-token kernel in verify mode) has recorded, per token t,
// the normalised key k_t, the write delta_t and the decay alpha_t, with which the gated
// delta rule of step 7 on the page "spark_model/forward/qwen3_5/linear_attention.rs"
// reads S_t = alpha_t S_{t-1} + k_t delta_t^T. Here the state the verify call read is
// streamed from HBM once, the n accepted updates are applied in order in registers,
// and the tile is written back once: the pass is bound by HBM bandwidth like a
// single-token step. The conv history (step 3) becomes the last W-1 raw inputs of
// [history, tokens 0..n-1], a bit copy. This is the GDN counterpart of rewinding a
// rejected speculative draft ("metrale_model_arch/glm5next_dsa/layer.rs", the lockstep
// check and rewind_to): the recurrent state cannot be truncated, so it is rebuilt from
// the recorded factors of the accepted prefix.
//
// One CTA per (sequence, v-head). A thread holds RPT consecutive rows x 4 columns of
// the dk x dv tile (one float4 per row), the TPR threads of a row segment covering it
// with whole sectors; two CTAs share an SM. The CTA of the first v-head of a k-head group also rolls that
// k-head's q and k channels; every CTA rolls its own v-head's v channels.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// A thread holds RPT rows x 4 columns (about 32 values): up to 512 threads per tile and
// two CTAs per SM, so one CTA's loads overlap the other's update and stores.
template <int DK, int DV>
struct CommitGeo {
    static constexpr int TPR = DV / 4;  // threads per row segment
    static constexpr int NT0 = DK * DV / 32;
    static constexpr int NT = NT0 < 32 ? 32 : (NT0 > 512 ? 512 : NT0);
    static constexpr int RPP = NT / TPR;
    static constexpr int RPT = DK / RPP;
    static_assert(NT % TPR == 0 && DK % RPP == 0 && RPT >= 1, "commit geometry");
};

template <int DK, int DV>
__global__ void __launch_bounds__(CommitGeo<DK, DV>::NT, 2)
spec_commit_kernel(const SpecCommitArgs p) {
    using Geo = CommitGeo<DK, DV>;
    constexpr int RPT = Geo::RPT, NT = Geo::NT;
    extern __shared__ __align__(16) float sm[];  // [T][DK] keys, [T][DV] writes, [T] decays
    const int Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk, W = p.sh.W, C = p.sh.C, T = p.T;
    const int seq = blockIdx.x / Hv, h = blockIdx.x - seq * Hv, hk = h / G;
    const int tid = threadIdx.x;

    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int n = __ldg(p.n_accept + seq);
    const int slot = __ldg(p.slots + seq);
    if (n < 0 || n > T) {
        if (tid == 0 && h == 0 && p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_SEQLEN_BIT);
        return;
    }
    if (slot < 0 || slot >= p.P) {
        if (tid == 0 && h == 0 && p.err_flag && n > 0) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        return;
    }
    if (n == 0) return;  // nothing accepted: the pools stay as they are

    // the state tile into registers first (the long-latency loads), then the factors
    const int cg = tid % Geo::TPR, row0 = (tid / Geo::TPR) * RPT;
    float4* Sg = reinterpret_cast<float4*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV)) +
                 (size_t)row0 * (DV / 4) + cg;
    float4 S[RPT];
#pragma unroll
    for (int s = 0; s < RPT; ++s) S[s] = __ldcs(Sg + (size_t)s * (DV / 4));
    float* ks = sm;
    float* ds = ks + T * DK;
    float* as = ds + T * DV;
    for (int i = tid; i < n * DK; i += NT) {
        const int t = i / DK, r = i - t * DK;
        ks[i] = p.spec_k[(((size_t)seq * T + t) * Hk + hk) * DK + r];
    }
    for (int i = tid; i < n * DV; i += NT) {
        const int t = i / DV, c = i - t * DV;
        ds[i] = p.spec_delta[(((size_t)seq * T + t) * Hv + h) * DV + c];
    }
    if (tid < n) as[tid] = p.spec_alpha[((size_t)seq * T + tid) * Hv + h];

    __syncthreads();

    // S <- alpha_t S + k_t delta_t^T for the accepted tokens, in order
    for (int t = 0; t < n; ++t) {
        const float al = as[t];
        const float4 d = reinterpret_cast<const float4*>(ds + t * DV)[cg];
        const float* kr = ks + t * DK + row0;
#pragma unroll
        for (int s = 0; s < RPT; ++s) {
            const float kv = kr[s];
            S[s].x = fmaf(al, S[s].x, kv * d.x);
            S[s].y = fmaf(al, S[s].y, kv * d.y);
            S[s].z = fmaf(al, S[s].z, kv * d.z);
            S[s].w = fmaf(al, S[s].w, kv * d.w);
        }
    }
#pragma unroll
    for (int s = 0; s < RPT; ++s) __stcs(Sg + (size_t)s * (DV / 4), S[s]);

    // the conv history of this CTA's channels: v-head h's v channels, and the k-head's
    // q and k channels in the group's first CTA. New row r is element n + r of
    // [history rows 0..W-2, tokens 0..T-1]; every value is read before any is written.
    {
        uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
        const uint16_t* x = p.qkv + (size_t)seq * T * C;
        const int nqk = h % G == 0 ? 2 * DK : 0;
        for (int i = tid; i < nqk + DV; i += NT) {
            const int ch = i >= nqk ? 2 * Hk * DK + h * DV + (i - nqk)  // v
                                    : (i < DK ? hk * DK + i : Hk * DK + hk * DK + (i - DK));  // q, k
            uint16_t nv[kMaxConvWidth - 1];
#pragma unroll
            for (int r = 0; r < kMaxConvWidth - 1; ++r) {
                const int e = n + r;
                nv[r] = r < W - 1 ? (e < W - 1 ? hist[(size_t)e * C + ch] : x[(size_t)(e - (W - 1)) * C + ch]) : 0;
            }
#pragma unroll
            for (int r = 0; r < kMaxConvWidth - 1; ++r)
                if (r < W - 1) hist[(size_t)r * C + ch] = nv[r];
        }
    }
}

template <int DK, int DV>
cudaError_t launch_commit(const SpecCommitArgs& a, cudaStream_t stream) {
    auto kern = spec_commit_kernel<DK, DV>;
    const size_t smem = (size_t)a.T * (DK + DV + 1) * sizeof(float);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.sh.Hv));
    cfg.blockDim = dim3(CommitGeo<DK, DV>::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int DK>
cudaError_t commit_dispatch(const SpecCommitArgs& a, cudaStream_t stream) {
    switch (a.sh.dv) {
        case 16: return launch_commit<DK, 16>(a, stream);
        case 32: return launch_commit<DK, 32>(a, stream);
        case 64: return launch_commit<DK, 64>(a, stream);
        case 128: return launch_commit<DK, 128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_spec_commit(const SpecCommitArgs& a, cudaStream_t stream) {
    if (a.B == 0) return cudaSuccess;
    switch (a.sh.dk) {
        case 16: return commit_dispatch<16>(a, stream);
        case 32: return commit_dispatch<32>(a, stream);
        case 64: return commit_dispatch<64>(a, stream);
        case 128: return commit_dispatch<128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gdn
