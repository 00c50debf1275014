// Fused GDN decode step for launches of several tokens per sequence (T = 2..16):
// steps 3 to 8 and the SiLU(z) gate of steps 9+10+11 on the page
// "spark_model/forward/qwen3_5/linear_attention.rs", applied to the tokens of the
// launch in order with the state kept on chip in between (the tokens of one launch
// behave exactly like T single-token calls).
//
// Work. One CTA per (sequence, v-head) h, with DV/16 warps. Each warp owns 16
// columns of the head's dk x dv state for the whole launch, in registers: lane
// (rg, cg) holds the four columns 16 w + 4 cg of the rows 32 j + 4 rg + e. The
// columns of S are independent under the update, so a warp needs nobody else inside
// the token loop: S^T k and S^T q reduce over the rows with three shuffle rounds, and
// the warps of a CTA meet only before the loop (conv and per-token scalars) and
// after it (the RMSNorm over the head).
//
// The decay is carried as a scale: the registers hold S~ with S = c S~, c the
// running product of the decays of this launch's tokens (reset to 1, with S~ scaled,
// whenever it would drop below 2^-64). The update of a token is then one FMA per
// element, S~ += k (nk delta / c), instead of a multiply and an FMA.
//
// The CTAs of one k-head's v-heads form a cluster: each recomputes the conv of the
// k-head's q/k channels from the same stored history, and the first rewrites that
// history only after the cluster barrier says every CTA has read it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kMtMaxTokens = 16;

// SiLU with the hardware exponential and an approximate division (relative error a
// few ulp; the multi-token conv evaluates it for every channel of every token).
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

template <int DK, int DV>
struct MtGeo {
    static constexpr int NW = DV / 16;           // warps: 16 columns each
    static constexpr int NT = 32 * NW;
    static constexpr int RG = 8, CG = 4;         // lanes: 8 row groups x 4 groups of four columns
    static constexpr int RPL = DK / RG;          // rows per lane
    static constexpr int NCH = 2 * DK + DV;      // conv channels of a CTA: q, k of the k-head, v of the head
    static_assert(DV % 16 == 0 && RPL >= 2 && (RPL == 2 || RPL % 4 == 0), "multi-token geometry");
    // Shared memory (bytes): staged raw rows (W-1 history rows, then T tokens) and the
    // channels' weights as bf16; then fp32 raw q/k and v per token, o per token and
    // the per-token scalars.
    static __host__ __device__ int rows_bytes(int W, int T) { return ((W - 1 + T) * NCH * 2 + 15) & ~15; }
    static __host__ __device__ int wts_off(int W, int T) { return rows_bytes(W, T); }
    static __host__ __device__ int qk_off(int W, int T) { return wts_off(W, T) + ((NCH * W * 2 + 15) & ~15); }
    static __host__ __device__ int vs_off(int W, int T) { return qk_off(W, T) + T * 2 * DK * 4; }
    static __host__ __device__ int os_off(int W, int T) { return vs_off(W, T) + T * DV * 4; }
    static __host__ __device__ int sc_off(int W, int T) { return os_off(W, T) + T * DV * 4; }
    static __host__ __device__ int total(int W, int T) { return sc_off(W, T) + T * (int)sizeof(TokenScalars); }
};

// Row held by lane row group rg in register block j, element e.
template <int RPL>
__device__ __forceinline__ int mt_row(int j, int rg, int e) {
    return RPL == 2 ? 2 * rg + e : 32 * j + 4 * rg + e;
}

template <int DK, int DV>
__global__ void __launch_bounds__(MtGeo<DK, DV>::NT, (MtGeo<DK, DV>::NT >= 256 ? 2 : 512 / MtGeo<DK, DV>::NT))
decode_mt_kernel(const DecodeArgs p) {
    using Geo = MtGeo<DK, DV>;
    constexpr int RPL = Geo::RPL, NCH = Geo::NCH, NB = RPL == 2 ? 1 : RPL / 4, EPB = RPL == 2 ? 2 : 4;
    extern __shared__ __align__(128) unsigned char smem[];
    const int T = p.T, W = p.sh.W, C = p.sh.C, Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk;
    const int seq = blockIdx.x / Hv, h = blockIdx.x - seq * Hv, hk = h / G, gi = h - hk * G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint16_t* rows = reinterpret_cast<uint16_t*>(smem);
    uint16_t* wts = reinterpret_cast<uint16_t*>(smem + Geo::wts_off(W, T));
    float* qk = reinterpret_cast<float*>(smem + Geo::qk_off(W, T));
    float* vs = reinterpret_cast<float*>(smem + Geo::vs_off(W, T));
    float* os = reinterpret_cast<float*>(smem + Geo::os_off(W, T));
    TokenScalars* sc = reinterpret_cast<TokenScalars*>(smem + Geo::sc_off(W, T));

    const int slot = __ldg(p.slots + seq);
    if (slot < 0 || slot >= p.P) {  // every CTA of the cluster has this sequence: they all leave
        if (tid == 0 && gi == 0 && p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
        return;
    }

    // ---- the state tile into registers (streamed: read once here, written once at the end)
    const int rg = lane >> 2, cg = lane & 3, col = 16 * warp + 4 * cg;
    float* Sg = p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV) + col;
    float4 S[RPL];
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int e = 0; e < EPB; ++e)
            S[j * EPB + e] = __ldcs(reinterpret_cast<const float4*>(Sg + (size_t)mt_row<RPL>(j, rg, e) * DV));

    // ---- stage the conv inputs: the slot's W-1 history rows, then the T tokens' raw
    // rows, for the CTA's three channel runs (q, k of the k-head, v of the head), and
    // the runs' weights. Every run is a multiple of 8 channels: 16-byte copies.
    const int ch_q = hk * DK, ch_k = Hk * DK + hk * DK, ch_v = 2 * Hk * DK + h * DV;
    auto run_channel = [&](int lc) { return lc < DK ? ch_q + lc : (lc < 2 * DK ? ch_k + lc - DK : ch_v + lc - 2 * DK); };
    const uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
    const uint16_t* x = p.qkv + (size_t)seq * T * C;
    const int nrow = W - 1 + T;
    for (int i = tid; i < nrow * (NCH / 8); i += Geo::NT) {
        const int r = i / (NCH / 8), lc = (i - r * (NCH / 8)) * 8, ch = run_channel(lc);
        const uint16_t* src = r < W - 1 ? hist + (size_t)r * C + ch : x + (size_t)(r - (W - 1)) * C + ch;
        *reinterpret_cast<uint4*>(rows + r * NCH + lc) = __ldg(reinterpret_cast<const uint4*>(src));
    }
    for (int i = tid; i < NCH * W / 8; i += Geo::NT) {  // weights [NCH][W]: three runs of consecutive channels
        const int lc = (i * 8) / W, off = i * 8 - lc * W;
        // a 16-byte group never straddles two runs: every run holds a multiple of 8 channels
        const int ch = run_channel(lc);
        *reinterpret_cast<uint4*>(wts + i * 8) =
            __ldg(reinterpret_cast<const uint4*>(p.conv_w + (size_t)ch * W + off));
    }
    // ---- steps 4, 5: decay and write strength of v-head h, per token
    if (tid < T) {
        const size_t i = ((size_t)seq * T + tid) * Hv + h;
        gate_and_beta(p.a[i], p.b[i], p.A_log[h], p.dt_bias[h], sc[tid].alpha, sc[tid].beta);
    }
    __syncthreads();
    if (G > 1) cluster_arrive_relaxed();  // this CTA has read the stored history

    // ---- step 3: conv + SiLU of every channel for every token. The window of the last
    // kMaxConvWidth staged rows slides through registers with the newest row at the
    // top, the weights aligned to it (taps beyond W are zero), so every register index
    // is a compile-time constant whatever W is.
    for (int lc = tid; lc < NCH; lc += Geo::NT) {
        float wr[kMaxConvWidth], win[kMaxConvWidth];
#pragma unroll
        for (int m = 0; m < kMaxConvWidth; ++m) {
            const int j = W - kMaxConvWidth + m;  // tap of window position m: it multiplies staged row t + j
            wr[m] = j >= 0 ? bf16_bits_to_float(wts[lc * W + j]) : 0.f;
            // before token 0's shift position m holds staged row j - 1 (history rows only)
            win[m] = j >= 1 ? bf16_bits_to_float(rows[(j - 1) * NCH + lc]) : 0.f;
        }
        for (int t = 0; t < T; ++t) {
#pragma unroll
            for (int m = 0; m < kMaxConvWidth - 1; ++m) win[m] = win[m + 1];
            win[kMaxConvWidth - 1] = bf16_bits_to_float(rows[(t + W - 1) * NCH + lc]);
            float u = 0.f;
#pragma unroll
            for (int m = 0; m < kMaxConvWidth; ++m) u = fmaf(wr[m], win[m], u);
            const float s = silu_fast(u);
            if (lc < 2 * DK) qk[t * 2 * DK + lc] = s;
            else vs[t * DV + lc - 2 * DK] = s;
        }
    }
    __syncthreads();
    // L2 norms of q and k (step 3) as factors on the raw values, and k.q
    qk_norms<DK>(qk, sc, T, p.sh.l2_eps, p.sh.q_scale, Geo::NW);
    __syncthreads();

    // ---- steps 6, 7: the recurrence, token by token, on this warp's columns
    float c = 1.f;  // S = c * S~ (the registers hold S~)
    for (int t = 0; t < T; ++t) {
        const float* qr = qk + t * 2 * DK;
        const float* kr = qr + DK;
        float kreg[RPL];
        float4 mk = make_float4(0.f, 0.f, 0.f, 0.f), mq = mk;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            float kk[EPB], qq[EPB];
            const int r0 = mt_row<RPL>(j, rg, 0);
            if constexpr (EPB == 4) {
                const float4 k4 = *reinterpret_cast<const float4*>(kr + r0);
                const float4 q4 = *reinterpret_cast<const float4*>(qr + r0);
                kk[0] = k4.x; kk[1] = k4.y; kk[2] = k4.z; kk[3] = k4.w;
                qq[0] = q4.x; qq[1] = q4.y; qq[2] = q4.z; qq[3] = q4.w;
            } else {
                const float2 k2 = *reinterpret_cast<const float2*>(kr + r0);
                const float2 q2 = *reinterpret_cast<const float2*>(qr + r0);
                kk[0] = k2.x; kk[1] = k2.y;
                qq[0] = q2.x; qq[1] = q2.y;
            }
#pragma unroll
            for (int e = 0; e < EPB; ++e) {
                const float4 s = S[j * EPB + e];
                kreg[j * EPB + e] = kk[e];
                mk.x = fmaf(s.x, kk[e], mk.x); mk.y = fmaf(s.y, kk[e], mk.y);
                mk.z = fmaf(s.z, kk[e], mk.z); mk.w = fmaf(s.w, kk[e], mk.w);
                mq.x = fmaf(s.x, qq[e], mq.x); mq.y = fmaf(s.y, qq[e], mq.y);
                mq.z = fmaf(s.z, qq[e], mq.z); mq.w = fmaf(s.w, qq[e], mq.w);
            }
        }
#pragma unroll
        for (int off = Geo::CG; off < 32; off <<= 1) {  // over the row groups (lanes with the same columns)
            mk.x += __shfl_xor_sync(0xffffffffu, mk.x, off); mk.y += __shfl_xor_sync(0xffffffffu, mk.y, off);
            mk.z += __shfl_xor_sync(0xffffffffu, mk.z, off); mk.w += __shfl_xor_sync(0xffffffffu, mk.w, off);
            mq.x += __shfl_xor_sync(0xffffffffu, mq.x, off); mq.y += __shfl_xor_sync(0xffffffffu, mq.y, off);
            mq.z += __shfl_xor_sync(0xffffffffu, mq.z, off); mq.w += __shfl_xor_sync(0xffffffffu, mq.w, off);
        }
        const TokenScalars st = sc[t];
        const float4 v = *reinterpret_cast<const float4*>(vs + t * DV + col);
        const float c1 = c * st.alpha;  // S after this token's decay is c1 * S~
        const float am = c1 * st.nk, aq = c1 * st.nq;
        float4 d, o;
        d.x = st.beta * fmaf(-am, mk.x, v.x); d.y = st.beta * fmaf(-am, mk.y, v.y);
        d.z = st.beta * fmaf(-am, mk.z, v.z); d.w = st.beta * fmaf(-am, mk.w, v.w);
        o.x = fmaf(aq, mq.x, d.x * st.kq); o.y = fmaf(aq, mq.y, d.y * st.kq);
        o.z = fmaf(aq, mq.z, d.z * st.kq); o.w = fmaf(aq, mq.w, d.w * st.kq);
        if (rg == 0) *reinterpret_cast<float4*>(os + t * DV + col) = o;
        float f;  // the update's factor on the raw k: nk delta / c, with c the new scale
        if (c1 < 0x1p-64f) {  // fold the scale into the registers before it underflows
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                S[i].x *= c1; S[i].y *= c1; S[i].z *= c1; S[i].w *= c1;
            }
            c = 1.f;
            f = st.nk;
        } else {
            c = c1;
            f = __fdividef(st.nk, c1);
        }
        const float4 dn = make_float4(d.x * f, d.y * f, d.z * f, d.w * f);
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            S[i].x = fmaf(kreg[i], dn.x, S[i].x); S[i].y = fmaf(kreg[i], dn.y, S[i].y);
            S[i].z = fmaf(kreg[i], dn.z, S[i].z); S[i].w = fmaf(kreg[i], dn.w, S[i].w);
        }
    }
    // the state back to the pool, scale applied
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int e = 0; e < EPB; ++e) {
            const float4 s = S[j * EPB + e];
            __stcs(reinterpret_cast<float4*>(Sg + (size_t)mt_row<RPL>(j, rg, e) * DV),
                   make_float4(s.x * c, s.y * c, s.z * c, s.w * c));
        }
    __syncthreads();

    // ---- step 8 over the head, the norm weight and SiLU(z): one warp per token, four
    // columns per lane (DV <= 128)
    const bool has_cols = 4 * lane < DV;
    const uint2 nw = has_cols ? __ldg(reinterpret_cast<const uint2*>(p.norm_w) + lane) : make_uint2(0u, 0u);
    for (int t = warp; t < T; t += Geo::NW) {
        const float4 o = has_cols ? reinterpret_cast<const float4*>(os + t * DV)[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
        float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (!has_cols) continue;
        const float inv = rsqrtf(ss / (float)DV + p.sh.rms_eps);
        const size_t base = (((size_t)seq * T + t) * Hv + h) * DV + 4 * lane;
        const uint2 zz = __ldg(reinterpret_cast<const uint2*>(p.z + base));
        const float y0 = o.x * inv * bf16_bits_to_float(nw.x & 0xffffu) * silu(bf16_bits_to_float(zz.x & 0xffffu));
        const float y1 = o.y * inv * bf16_bits_to_float(nw.x >> 16) * silu(bf16_bits_to_float(zz.x >> 16));
        const float y2 = o.z * inv * bf16_bits_to_float(nw.y & 0xffffu) * silu(bf16_bits_to_float(zz.y & 0xffffu));
        const float y3 = o.w * inv * bf16_bits_to_float(nw.y >> 16) * silu(bf16_bits_to_float(zz.y >> 16));
        uint2 packed;
        packed.x = (uint32_t)float_to_bf16_bits(y0) | ((uint32_t)float_to_bf16_bits(y1) << 16);
        packed.y = (uint32_t)float_to_bf16_bits(y2) | ((uint32_t)float_to_bf16_bits(y3) << 16);
        *reinterpret_cast<uint2*>(p.out + base) = packed;
        if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + base) = make_float4(y0, y1, y2, y3);
    }

    // ---- the new conv history: the last W-1 raw inputs. The q/k channels are shared
    // by the cluster and rewritten by its first CTA once every CTA has read them.
    if (G > 1) cluster_wait_acquire();
    uint16_t* hw = p.conv_pool + (size_t)slot * (W - 1) * C;
    const int lc0 = (G == 1 || gi == 0) ? 0 : 2 * DK;
    const int nvec = (NCH - lc0) / 8;
    for (int i = tid; i < (W - 1) * nvec; i += Geo::NT) {
        const int r = i / nvec, lc = lc0 + (i - r * nvec) * 8;
        *reinterpret_cast<uint4*>(hw + (size_t)r * C + run_channel(lc)) =
            *reinterpret_cast<const uint4*>(rows + (T + r) * NCH + lc);
    }
}

template <int DK, int DV>
cudaError_t launch_mt(const DecodeArgs& a, cudaStream_t stream) {
    using Geo = MtGeo<DK, DV>;
    auto kern = decode_mt_kernel<DK, DV>;
    const int smem = Geo::total(a.sh.W, a.T);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.sh.Hv));
    cfg.blockDim = dim3(Geo::NT);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)(a.sh.Hv / a.sh.Hk);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int DK>
cudaError_t mt_dispatch(const DecodeArgs& a, cudaStream_t stream) {
    switch (a.sh.dv) {
        case 16: return launch_mt<DK, 16>(a, stream);
        case 32: return launch_mt<DK, 32>(a, stream);
        case 64: return launch_mt<DK, 64>(a, stream);
        case 128: return launch_mt<DK, 128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool multitoken_supported(const DecodeArgs& a) {
    return a.T >= 1 && a.T <= kMtMaxTokens && a.sh.Hv / a.sh.Hk <= 8 && a.sh.dv >= 16;
}

cudaError_t launch_decode_multitoken(const DecodeArgs& a, cudaStream_t stream) {
    switch (a.sh.dk) {
        case 16: return mt_dispatch<16>(a, stream);
        case 32: return mt_dispatch<32>(a, stream);
        case 64: return mt_dispatch<64>(a, stream);
        case 128: return mt_dispatch<128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gdn
