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
// A persistent CTA per SM streams the (sequence, v-head) units; for each, the CTA of the
// unit rolls the v-head's v channels, and the k-head's q and k channels for the first
// v-head of a group.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

// Persistent form: one CTA per SM walks the (sequence, v-head) units with an accepted
// token, cid, cid + grid, ...; a 2-stage ring in shared memory holds each unit's state
// tile and its factors, brought in by bulk copies (issued by warp 0, one copy per lane)
// while the CTA updates the previous unit. A thread holds RPT rows x 4 columns.
template <int DK, int DV>
struct CommitGeo {
    static constexpr int NT = 256;
    static constexpr int TPR = DV / 4;  // threads per row segment
    static constexpr int RPP = NT / TPR;
    static constexpr int RPT = DK / RPP < 1 ? 1 : DK / RPP;
    static constexpr int ACTIVE = RPP * RPT >= DK ? (DK / RPT) * TPR : NT;  // threads holding rows
    static constexpr int TILE = DK * DV * 4;
    static __host__ __device__ int stage_bytes(int T) { return TILE + T * (DK + DV) * 4; }
    static __host__ __device__ int smem_bytes(int T) { return 2 * stage_bytes(T) + 64; }
    static_assert(DV % 4 == 0 && NT % TPR == 0, "commit geometry");
};

template <int DK, int DV>
__global__ void __launch_bounds__(CommitGeo<DK, DV>::NT, 1)
spec_commit_kernel(const SpecCommitArgs p) {
    using Geo = CommitGeo<DK, DV>;
    constexpr int RPT = Geo::RPT, NT = Geo::NT;
    extern __shared__ __align__(128) unsigned char smem[];
    const int Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk, W = p.sh.W, C = p.sh.C, T = p.T;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sbytes = Geo::stage_bytes(T);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * sbytes);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 2);
    const int nunits = p.B * Hv;

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(full + 1, 1);
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    // The next unit of this CTA with an accepted token, from unit index u on (nunits:
    // none). Sequences with a count outside [0, T] or a slot out of range are flagged
    // once, by the CTA holding their first v-head.
    auto next_unit = [&](int u, int& n, int& slot) {
        for (; u < nunits; u += gridDim.x) {
            const int seq = u / Hv;
            n = __ldg(p.n_accept + seq);
            slot = __ldg(p.slots + seq);
            const bool bad_n = n < 0 || n > T, bad_slot = slot < 0 || slot >= p.P;
            if ((bad_n || (bad_slot && n > 0)) && u % Hv == 0 && tid == 0 && p.err_flag)
                atomicOr(p.err_flag, bad_n ? GDN_DEVICE_ERR_SEQLEN_BIT : GDN_DEVICE_ERR_SLOT_RANGE_BIT);
            if (!bad_n && !bad_slot && n > 0) return u;
        }
        return nunits;
    };
    // warp 0: the copies of unit u (accepted count n, slot) into stage s
    auto issue = [&](int s, int u, int n, int slot) {
        const int seq = u / Hv, h = u - seq * Hv, hk = h / G;
        unsigned char* st = smem + s * sbytes;
        if (lane == 0) mbar_arrive_expect_tx(full + s, (uint32_t)(Geo::TILE + n * (DK + DV) * 4));
        __syncwarp();
        constexpr int kChunks = Geo::TILE >= 16384 ? Geo::TILE / 16384 : 1;
        constexpr int kChunkBytes = Geo::TILE / kChunks;
        const char* tile = reinterpret_cast<const char*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV));
        for (int c = lane; c < kChunks + 2 * n; c += 32) {
            if (c < kChunks) {
                tma_load_1d(st + c * kChunkBytes, tile + c * kChunkBytes, kChunkBytes, full + s);
            } else if (c < kChunks + n) {
                const int t = c - kChunks;
                tma_load_1d(st + Geo::TILE + t * DK * 4, p.spec_k + (((size_t)seq * T + t) * Hk + hk) * DK, DK * 4,
                            full + s);
            } else {
                const int t = c - kChunks - n;
                tma_load_1d(st + Geo::TILE + T * DK * 4 + t * DV * 4,
                            p.spec_delta + (((size_t)seq * T + t) * Hv + h) * DV, DV * 4, full + s);
            }
        }
    };

    int n0 = 0, s0 = 0, n1 = 0, s1 = 0;
    int u0 = next_unit((int)blockIdx.x, n0, s0);
    int u1 = u0 < nunits ? next_unit(u0 + (int)gridDim.x, n1, s1) : nunits;
    if (warp == 0) {
        if (u0 < nunits) issue(0, u0, n0, s0);
        if (u1 < nunits) issue(1, u1, n1, s1);
    }
    const int cg = tid % Geo::TPR, row0 = (tid / Geo::TPR) * RPT;
    const bool holds = tid < Geo::ACTIVE;
    int drain_j = -1, drain_next = 0;  // on a timeout: the unit whose wait gave up, and whether one more was issued
    for (int j = 0; u0 < nunits; ++j) {
        const int s = j & 1, seq = u0 / Hv, h = u0 - seq * Hv, hk = h / G, n = n0, slot = s0;
        const bool ok = mbar_wait_deadline(full + s, (uint32_t)((j >> 1) & 1), kWaitTimeoutCycles,
                                           [&] { return *abort_flag != 0; });
        if (!__syncthreads_and(ok)) {
            if (tid == 0) {
                *abort_flag = 1;
                if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
            }
            drain_j = j;
            drain_next = u1 < nunits;
            break;
        }
        const unsigned char* st = smem + s * sbytes;
        const float* ks = reinterpret_cast<const float*>(st + Geo::TILE);
        const float* ds = ks + T * DK;
        if (holds) {
            // S <- alpha_t S + k_t delta_t^T for the accepted tokens, in order, from the staged
            // tile; the rows go straight to the pool
            const float4* tl = reinterpret_cast<const float4*>(st) + (size_t)row0 * (DV / 4) + cg;
            float4 S[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) S[r] = tl[(size_t)r * (DV / 4)];
            for (int t = 0; t < n; ++t) {
                const float al = __ldg(p.spec_alpha + ((size_t)seq * T + t) * Hv + h);
                const float4 d = reinterpret_cast<const float4*>(ds + t * DV)[cg];
                const float* kr = ks + t * DK + row0;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const float kv = kr[r];
                    S[r].x = fmaf(al, S[r].x, kv * d.x);
                    S[r].y = fmaf(al, S[r].y, kv * d.y);
                    S[r].z = fmaf(al, S[r].z, kv * d.z);
                    S[r].w = fmaf(al, S[r].w, kv * d.w);
                }
            }
            float4* Sg = reinterpret_cast<float4*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV)) +
                         (size_t)row0 * (DV / 4) + cg;
#pragma unroll
            for (int r = 0; r < RPT; ++r) __stcs(Sg + (size_t)r * (DV / 4), S[r]);
        }
        // the conv history of this unit's channels: v-head h's v channels, and the k-head's q
        // and k channels in the group's first v-head. New row r is element n + r of
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
        __syncthreads();  // every read of stage s is done: it takes the unit after next
        int n2 = 0, s2 = 0;
        const int u2 = u1 < nunits ? next_unit(u1 + (int)gridDim.x, n2, s2) : nunits;
        if (warp == 0 && u2 < nunits) {
            fence_proxy_async_smem();  // the stage's generic reads before the copies overwrite it
            issue(s, u2, n2, s2);
        }
        u0 = u1; n0 = n1; s0 = s1;
        u1 = u2; n1 = n2; s1 = s2;
    }
    // After a timeout the copies in flight land before the CTA leaves: those of the unit
    // whose wait gave up and, if it was issued, of the next one (each phase counts its
    // copies; no other phase is armed).
    if (drain_j >= 0 && tid == 0) {
        mbar_wait_bounded(full + (drain_j & 1), (uint32_t)((drain_j >> 1) & 1));
        if (drain_next) mbar_wait_bounded(full + ((drain_j + 1) & 1), (uint32_t)(((drain_j + 1) >> 1) & 1));
    }
}

template <int DK, int DV>
cudaError_t launch_commit(const SpecCommitArgs& a, cudaStream_t stream) {
    using Geo = CommitGeo<DK, DV>;
    auto kern = spec_commit_kernel<DK, DV>;
    const int smem = Geo::smem_bytes(a.T);
    static std::mutex mu;
    static int sms_cache[kMaxDevices];
    static int attr_set[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (attr_set[dev] < smem) {
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          Geo::smem_bytes(kMaxTokens))) != cudaSuccess)
                return e;
            attr_set[dev] = Geo::smem_bytes(kMaxTokens);
        }
        if (sms_cache[dev] <= 0 &&
            (e = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        sms = sms_cache[dev];
    }
    const int units = a.B * a.sh.Hv;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units < sms ? units : sms));
    cfg.blockDim = dim3(Geo::NT);
    cfg.dynamicSmemBytes = (size_t)smem;
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
