// Persistent, software-pipelined form of the fused GDN decode step for single-token
// launches over many sequences (steps 3 to 8 and the SiLU(z) gate of steps 9+10+11
// on the page "spark_model/forward/qwen3_5/linear_attention.rs").
//
// A cluster of G = Hv/Hk CTAs (one per v-head sharing a k-head) stays resident and
// walks (sequence, k-head) groups cid, cid + ncl, cid + 2 ncl, ... Each CTA owns one
// v-head of the group: its whole dk x dv fp32 state tile, which is contiguous in the
// pool. Tiles stream through a ring of NSTAGE shared-memory stages filled by TMA bulk
// copies, so while unit u is computed the tiles of units u+1 .. u+NSTAGE-1 are in
// flight and the updated tile of unit u-1 drains from registers: the SM keeps HBM
// busy instead of alternating between load, compute and store phases.
//
// Conv ownership: the group's q and k channels are split over the G CTAs and each
// CTA owns its v-head's v channels, so every channel's history is read and rolled
// by exactly one CTA. The raw q/k values travel to every CTA of the cluster with
// st.async into distributed shared memory, completed on the receiver's mbarrier
// (no release fence that would wait for this CTA's outstanding state stores). The
// conv inputs of unit u+1 are loaded into registers while unit u is computed.
//
// Every wait is an mbarrier poll with a bound; on expiry the CTA sets the timeout
// bit of the error flag, stops issuing copies, waits (bounded) for the copies it
// has in flight and leaves through the final cluster barrier.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr uint32_t kPollLimit = 1u << 24;
constexpr int kTileChunk = 16384;  // bytes per bulk copy of a state tile

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int DK, int DV>
struct PLayout {
    using Geo = Tile<DK, DV>;
    static constexpr int NT = Geo::NT;
    static constexpr int TILE_BYTES = DK * DV * 4;
    static constexpr int NSTAGE = TILE_BYTES * 4 <= 196608 ? 4 : (TILE_BYTES * 3 <= 196608 ? 3 : 2);
    // most channels one CTA convolves: all 2*DK q/k channels (G = 1) plus its DV v channels
    static constexpr int MAXC = (2 * DK + DV + NT - 1) / NT;
    static constexpr int TILES = 0;
    static constexpr int ZB = TILES + NSTAGE * TILE_BYTES;       // [NSTAGE][DV] bf16
    static constexpr int QK = ZB + round_up(NSTAGE * DV * 2, 16);  // [2][2*DK] f32, raw q then raw k
    static constexpr int VS = QK + 2 * 2 * DK * 4;                // [2][DV] f32
    static constexpr int OS = VS + 2 * DV * 4;                    // [DV] f32
    static constexpr int RED = OS + DV * 4;                       // [2][NW][2][DV] f32
    static constexpr int SC = RED + 2 * Geo::NW * 2 * DV * 4;     // [2] TokenScalars
    static constexpr int PART = SC + 48;                          // [NW] f32
    static constexpr int BARS = round_up(PART + Geo::NW * 4, 16);  // [NSTAGE] tile bars, [2] q/k bars
    static constexpr int TOTAL = BARS + (NSTAGE + 2) * 8;
    static_assert(TOTAL <= 232448, "shared memory");
};

template <int DK, int DV>
__global__ void __launch_bounds__(PLayout<DK, DV>::NT, 1)
decode_persistent_kernel(const DecodeArgs p, const int ncl) {
    using Lay = PLayout<DK, DV>;
    using Geo = Tile<DK, DV>;
    constexpr int NT = Lay::NT, NSTAGE = Lay::NSTAGE, MAXC = Lay::MAXC, WM = kMaxConvWidth;
    extern __shared__ __align__(128) unsigned char smem[];
    float* tiles = reinterpret_cast<float*>(smem + Lay::TILES);
    uint16_t* zb = reinterpret_cast<uint16_t*>(smem + Lay::ZB);
    float* qkb = reinterpret_cast<float*>(smem + Lay::QK);
    float* vsb = reinterpret_cast<float*>(smem + Lay::VS);
    float* os = reinterpret_cast<float*>(smem + Lay::OS);
    float* red = reinterpret_cast<float*>(smem + Lay::RED);
    TokenScalars* scb = reinterpret_cast<TokenScalars*>(smem + Lay::SC);
    float* part = reinterpret_cast<float*>(smem + Lay::PART);
    uint64_t* tbar = reinterpret_cast<uint64_t*>(smem + Lay::BARS);
    uint64_t* qbar = tbar + NSTAGE;

    const int Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk, C = p.sh.C, W = p.sh.W;
    const int rank = (int)cluster_ctarank(), cid = blockIdx.x / G;
    const int ngroups = p.B * Hk;
    const int n = cid < ngroups ? (ngroups - cid + ncl - 1) / ncl : 0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int qk_lo = (rank * 2 * DK) / G, qk_hi = ((rank + 1) * 2 * DK) / G, nqk = qk_hi - qk_lo;
    const int nch = nqk + DV;

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(tbar + s, 1);
        mbar_init(qbar + 0, 1);
        mbar_init(qbar + 1, 1);
        mbar_init_fence();
    }
    __syncthreads();
    cluster_arrive_relaxed();  // every CTA of the cluster runs before any st.async targets it
    cluster_wait_acquire();

    auto group_seq = [&](int u) { return (cid + u * ncl) / Hk; };
    auto group_hk = [&](int u) { return (cid + u * ncl) % Hk; };
    auto slot_ok = [&](int s) { return s >= 0 && s < p.P; };
    auto slot_of = [&](int u) { return u < n ? __ldg(p.slots + group_seq(u)) : -1; };

    // thread 0: stage unit u's state tile and its z row into stage u % NSTAGE
    auto issue_tile = [&](int u) {
        const int seq = group_seq(u), h = group_hk(u) * G + rank;
        const int slot = __ldg(p.slots + seq);
        uint64_t* bar = tbar + (u % NSTAGE);
        if (!slot_ok(slot)) {
            mbar_arrive(bar);
            return;
        }
        mbar_arrive_expect_tx(bar, Lay::TILE_BYTES + DV * 2);
        const char* src = reinterpret_cast<const char*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV));
        char* dst = reinterpret_cast<char*>(tiles) + (size_t)(u % NSTAGE) * Lay::TILE_BYTES;
        for (int c = 0; c < Lay::TILE_BYTES; c += kTileChunk)
            tma_load_1d(dst + c, src + c, (uint32_t)min(kTileChunk, Lay::TILE_BYTES - c), bar);
        tma_load_1d(zb + (u % NSTAGE) * DV, p.z + ((size_t)seq * Hv + h) * DV, DV * 2, bar);
    };

    // conv inputs of one unit, one channel per (thread, i)
    uint32_t ph[MAXC][WM - 1], px[MAXC], pw[MAXC][WM];
    uint16_t pa = 0, pb = 0;
    float pA = 0.f, pdt = 0.f;
    auto channel_of = [&](int c, int hk, int h) {
        if (c < nqk) {
            const int j = qk_lo + c;
            return j < DK ? hk * DK + j : Hk * DK + hk * DK + (j - DK);
        }
        return 2 * Hk * DK + h * DV + (c - nqk);
    };
    auto prefetch = [&](int u, int slot) {
        const int seq = group_seq(u), hk = group_hk(u), h = hk * G + rank;
        const uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int c = tid + i * NT;
            if (c < nch) {
                const int ch = channel_of(c, hk, h);
#pragma unroll
                for (int r = 0; r < WM - 1; ++r) ph[i][r] = r < W - 1 ? hist[(size_t)r * C + ch] : 0u;
                px[i] = p.qkv[(size_t)seq * C + ch];
#pragma unroll
                for (int j = 0; j < WM; ++j) pw[i][j] = j < W ? p.conv_w[(size_t)ch * W + j] : 0u;
            }
        }
        if (tid == 0) {
            pa = p.a[(size_t)seq * Hv + h];
            pb = p.b[(size_t)seq * Hv + h];
            pA = p.A_log[h];
            pdt = p.dt_bias[h];
        }
    };
    // step 3 for unit u from the prefetched inputs: q/k shares to every cluster CTA,
    // v to this CTA, the rolled history back to the pool
    auto conv_finish = [&](int u, int slot) {
        const int hk = group_hk(u), h = hk * G + rank, buf = u & 1;
        uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int c = tid + i * NT;
            if (c < nch) {
                const int ch = channel_of(c, hk, h);
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < WM; ++j) {
                    if (j < W) {
                        const uint32_t xb = j < W - 1 ? ph[i][j] : px[i];
                        acc = fmaf(bf16_bits_to_float(pw[i][j]), bf16_bits_to_float(xb), acc);
                    }
                }
                const float s = silu(acc);
                if (c < nqk) {
                    const uint32_t a_loc = smem_addr(qkb + buf * 2 * DK + qk_lo + c);
                    const uint32_t b_loc = smem_addr(qbar + buf);
                    for (int r = 0; r < G; ++r) st_async_f32(cluster_map_u32(a_loc, r), s, cluster_map_u32(b_loc, r));
                } else {
                    vsb[buf * DV + (c - nqk)] = s;
                }
#pragma unroll
                for (int r = 0; r < WM - 1; ++r) {
                    if (r < W - 1) {
                        uint32_t nb = px[i];
                        if (r + 1 < WM - 1 && r + 1 < W - 1) nb = ph[i][r + 1 < WM - 1 ? r + 1 : 0];
                        hist[(size_t)r * C + ch] = (uint16_t)nb;
                    }
                }
            }
        }
    };

    int issued = 0;
    if (tid == 0)
        for (; issued < NSTAGE && issued < n; ++issued) issue_tile(issued);
    int slot_c = slot_of(0), slot_n1 = slot_of(1);
    if (n > 0 && slot_ok(slot_c)) {
        prefetch(0, slot_c);
        conv_finish(0, slot_c);
    } else if (n > 0 && tid == 0 && p.err_flag) {
        atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
    }
    uint16_t ga = pa, gb = pb;
    float gA = pA, gdt = pdt;

    bool failed = false;
    int consumed = 0;
    for (int u = 0; u < n; ++u) {
        const bool valid = slot_ok(slot_c);
        const int slot_n2 = slot_of(u + 2);
        if (u + 1 < n && slot_ok(slot_n1)) prefetch(u + 1, slot_n1);

        // ---- q/k of unit u have arrived from every cluster CTA: norms and gates
        const int buf = u & 1;
        if (tid == 0) {
            if (valid) mbar_arrive_expect_tx(qbar + buf, 2 * DK * 4);
            else mbar_arrive(qbar + buf);
        }
        bool ok = mbar_wait_bounded(qbar + buf, (u >> 1) & 1, kPollLimit);
        if (valid) {
            if (warp == 0) qk_norms<DK>(qkb + buf * 2 * DK, scb + buf, 1, p.sh.l2_eps, p.sh.q_scale, 1);
            if (tid == 0) gate_and_beta(ga, gb, gA, gdt, scb[buf].alpha, scb[buf].beta);
        }
        // ---- the state tile of unit u
        ok = mbar_wait_bounded(tbar + (u % NSTAGE), (u / NSTAGE) & 1, kPollLimit) && ok;
        ++consumed;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        const int seq = group_seq(u), h = group_hk(u) * G + rank;
        if (valid) {
            const int cg = tid % Geo::TPR, rp = tid / Geo::TPR;
            float4* Sg = reinterpret_cast<float4*>(p.state_pool + ((size_t)slot_c * Hv + h) * (size_t)(DK * DV)) +
                         (size_t)(rp * Geo::RPT) * (DV / 4) + cg;
            delta_rule_smem<DK, DV>(tiles + (size_t)(u % NSTAGE) * (DK * DV), qkb + buf * 2 * DK, vsb + buf * DV,
                                    scb + buf, os, red, 1, Sg, DV / 4);
        } else if (tid == 0 && p.err_flag) {
            atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        }
        __syncthreads();
        // ---- step 8: RMSNorm over the head, norm weight, SiLU(z) gate
        if (valid) {
            float ss = 0.f;
            for (int j = tid; j < DV; j += NT) ss = fmaf(os[j], os[j], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (lane == 0) part[warp] = ss;
            __syncthreads();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < Geo::NW; ++w) tot += part[w];
            const float inv = rsqrtf(tot / (float)DV + p.sh.rms_eps);
            for (int j = tid; j < DV; j += NT) {
                const float zz = bf16_bits_to_float(zb[(u % NSTAGE) * DV + j]);
                const float y = os[j] * inv * bf16_bits_to_float(p.norm_w[j]) * silu(zz);
                const size_t oi = ((size_t)seq * Hv + h) * DV + j;
                p.out[oi] = float_to_bf16_bits(y);
                if (p.out_f32) p.out_f32[oi] = y;
            }
        }
        __syncthreads();  // stage u % NSTAGE and its z row are free again
        if (tid == 0 && issued < n) {
            fence_proxy_async_smem();
            issue_tile(issued++);
        }
        if (u + 1 < n && slot_ok(slot_n1)) conv_finish(u + 1, slot_n1);
        ga = pa;  // the prefetched inputs of unit u+1 have long arrived by now
        gb = pb;
        gA = pA;
        gdt = pdt;
        slot_c = slot_n1;
        slot_n1 = slot_n2;
    }
    if (failed) {
        if (tid == 0) {
            if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
            for (int u = consumed; u < issued; ++u) mbar_wait_bounded(tbar + (u % NSTAGE), (u / NSTAGE) & 1, kPollLimit);
        }
        __syncthreads();
    }
    cluster_arrive_release();  // no CTA leaves while a peer may still send to it
    cluster_wait_acquire();
}

template <int DK, int DV>
cudaError_t launch_persistent_tile(const DecodeArgs& a, int G, cudaStream_t stream, bool query_only, int* cap_out) {
    using Lay = PLayout<DK, DV>;
    auto kern = decode_persistent_kernel<DK, DV>;
    // co-resident cluster capacity, queried once per (device, cluster size)
    static int cap_cache[16][9];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(Lay::NT);
    cfg.dynamicSmemBytes = Lay::TOTAL;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int& cap = cap_cache[dev & 15][G & 7 ? G : 8];
    if (cap <= 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::TOTAL);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3((unsigned)G);
        int maxc = 0;
        e = cudaOccupancyMaxActiveClusters(&maxc, kern, &cfg);
        if (e != cudaSuccess) return e;
        cap = maxc;
    }
    if (cap_out) *cap_out = cap;
    if (query_only) return cudaSuccess;
    const int ngroups = a.B * a.sh.Hk;
    const int ncl = ngroups < cap ? ngroups : cap;
    if (ncl <= 0) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)(ncl * G));
    return cudaLaunchKernelEx(&cfg, kern, a, ncl);
}

template <int DK>
cudaError_t persistent_dispatch(const DecodeArgs& a, int G, cudaStream_t stream, bool query_only, int* cap) {
    switch (a.sh.dv) {
        case 16: return launch_persistent_tile<DK, 16>(a, G, stream, query_only, cap);
        case 32: return launch_persistent_tile<DK, 32>(a, G, stream, query_only, cap);
        case 64: return launch_persistent_tile<DK, 64>(a, G, stream, query_only, cap);
        case 128: return launch_persistent_tile<DK, 128>(a, G, stream, query_only, cap);
    }
    return cudaErrorInvalidValue;
}

cudaError_t persistent_call(const DecodeArgs& a, cudaStream_t stream, bool query_only, int* cap) {
    const int G = a.sh.Hv / a.sh.Hk;
    switch (a.sh.dk) {
        case 16: return persistent_dispatch<16>(a, G, stream, query_only, cap);
        case 32: return persistent_dispatch<32>(a, G, stream, query_only, cap);
        case 64: return persistent_dispatch<64>(a, G, stream, query_only, cap);
        case 128: return persistent_dispatch<128>(a, G, stream, query_only, cap);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t persistent_capacity(const DecodeArgs& a, int* max_clusters) {
    return persistent_call(a, nullptr, true, max_clusters);
}

cudaError_t launch_decode_persistent(const DecodeArgs& a, cudaStream_t stream) {
    return persistent_call(a, stream, false, nullptr);
}

}  // namespace gdn
