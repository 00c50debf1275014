// Fused GDN decode step for launches of several tokens per sequence (up to 16):
// steps 3 to 8 and the SiLU(z) gate of steps 9+10+11 on the page
// "spark_model/forward/qwen3_5/linear_attention.rs", applied to the tokens of the
// launch in order with the state kept on chip in between (the tokens of one launch
// behave exactly like single-token calls, one per token). Every sequence has T tokens,
// or, with per-sequence offsets into packed rows, its own count up to T (none: the
// sequence is left as it is).
//
// Work. Persistent CTAs, one per SM, walk the (sequence, k-head) groups cid,
// cid + grid, ... A group's G v-heads are taken NH at a time (a "pass"); a pass
// holds NH v-heads with DV/16 warps each. Each warp owns 16 columns of its head's
// dk x dv state for the whole launch, in registers: lane (rg, cg) holds the four
// columns 16 w + 4 cg of the rows 32 j + 4 rg + e, as pairs of consecutive rows
// (S[r][c], S[r+1][c]) so that a 16-byte load of the raw k (or q) gives the packed
// FMA its (k_r, k_r+1) operands directly. The columns of S are independent under the
// update, so a warp needs nobody else inside the token loop: S^T k and S^T q reduce
// over the rows with three shuffle rounds.
//
// Pipelining. The inputs of the next pass (its NH state tiles, the conv history rows,
// the T raw token rows and the conv weights of its channels) travel by TMA bulk
// copies into one shared-memory stage while the current pass runs its tokens from
// registers; a pass empties the stage (state into registers, conv done, history
// rolled) before the next copies are issued. The state tiles travel as TMA bulk
// copies; the many short runs of raw rows and weights as 16-byte asynchronous copies
// spread over all threads, completing on the same barrier. The pass's z rows come the
// same way into their own buffer when the pass starts, and are read by its RMSNorm. A group's passes run back to back in
// one CTA, and the q/k conv history it shares is rewritten only by its last pass, so
// no other CTA ever reads a history this launch has written.
//
// The decay is carried as a scale: the registers hold S~ with S = c S~, c the
// running product of the decays of this launch's tokens (reset to 1, with S~ scaled,
// whenever it would drop below 2^-64). The update of a token is then one fused
// multiply-add per element, S~ += k (nk delta / c), done on pairs of columns with the
// packed FP32 instructions.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kMtMaxTokens = 16;
constexpr int kMtChunk = 16384;  // bytes per bulk copy of a state tile

// Two fp32 lanes in one 64-bit register pair, for the packed FP32 instructions of
// sm_100 (fma/mul .rn.f32x2: each lane rounds exactly like the scalar form).
typedef unsigned long long f2;
__device__ __forceinline__ f2 f2_pack(float a, float b) {
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(f2 v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ f2 f2_fma(f2 a, f2 b, f2 c) {  // a * b + c per lane
    f2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f2 f2_mul(f2 a, f2 b) {
    f2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// SiLU with the hardware exponential and an approximate division (relative error a
// few ulp; evaluated for every conv channel and every output element of every token).
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// Tokens of the recurrence taken together (a chunk); the on-chip buffers hold a whole
// number of chunks, the tokens past a sequence's last one being zero.
constexpr int kChunk = 4;
// Per (v-head, chunk): the scalars of the chunked recurrence (see the token loop).
constexpr int kCoefFloats = 36;
// Per token: raw k.k and k.q against the tokens of its chunk, and q.q.
constexpr int kGramFloats = 12;

template <int DK, int DV>
struct MtGeo {
    static constexpr int NWH = DV / 16;                       // warps per v-head: 16 columns each
    static constexpr int NHC = 16 / NWH < 8 ? 16 / NWH : 8;    // most v-heads one pass holds
    static constexpr int NW = NWH * NHC;
    static constexpr int NT = 32 * NW;
    static constexpr int RG = 8, CG = 4;                       // lanes: 8 row groups x 4 groups of four columns
    static constexpr int RPL = DK / RG;                        // rows per lane
    static constexpr int NCHC = 2 * DK + NHC * DV;             // most conv channels of a pass
    static constexpr int TILE = DK * DV * 4;
    static_assert(DV % 16 == 0 && RPL >= 2 && (RPL == 2 || RPL % 4 == 0), "multi-token geometry");
    static __host__ __device__ int padded(int T) { return (T + kChunk - 1) / kChunk * kChunk; }
    // Shared memory (bytes, every block 16-byte aligned): the stage (NHC state tiles,
    // the staged raw rows and the weights), then the raw q and k per token, v per v-head
    // and token (replaced by o: the warp that reads v_t of a column writes o_t of it),
    // the z rows of the pass, the per-token scalars, the Gram entries, the chunk
    // coefficients, the stage's slot and the abort flag, and the stage and z barriers.
    // Token buffers hold padded(T) tokens.
    static __host__ __device__ int rows_off() { return NHC * TILE; }
    static __host__ __device__ int wts_off(int W, int T) { return rows_off() + ((W - 1 + T) * NCHC * 2 + 15) / 16 * 16; }
    static __host__ __device__ int qk_off(int W, int T) { return wts_off(W, T) + (NCHC * W * 2 + 15) / 16 * 16; }
    static __host__ __device__ int vs_off(int W, int T) { return qk_off(W, T) + padded(T) * 2 * DK * 4; }
    static __host__ __device__ int zb_off(int W, int T) { return vs_off(W, T) + padded(T) * NHC * DV * 4; }
    static __host__ __device__ int sc_off(int W, int T) { return zb_off(W, T) + T * NHC * DV * 2; }
    static __host__ __device__ int gram_off(int W, int T) {
        return (sc_off(W, T) + padded(T) * NHC * (int)sizeof(TokenScalars) + 15) / 16 * 16;
    }
    static __host__ __device__ int coef_off(int W, int T) { return gram_off(W, T) + padded(T) * kGramFloats * 4; }
    static __host__ __device__ int dsm_off(int W, int T) {
        return coef_off(W, T) + NHC * (padded(T) / kChunk) * kCoefFloats * 4;
    }
    // per warp: the writes delta of the current chunk's tokens on its 16 columns
    static __host__ __device__ int ctl_off(int W, int T) { return dsm_off(W, T) + NW * kChunk * 16 * 4; }
    static __host__ __device__ int total(int W, int T) { return ctl_off(W, T) + 32; }
    // the control block: the stage's slot, the abort flag, the stage and z barriers,
    // the stage's first packed row and token count
};

template <int K>
struct Taps {  // a conv window of K taps, as a type
    static constexpr int value = K;
};

// Row held by lane row group rg in register block j, element e.
template <int RPL>
__device__ __forceinline__ int mt_row(int j, int rg, int e) {
    return RPL == 2 ? 2 * rg + e : 32 * j + 4 * rg + e;
}

template <int DK, int DV>
__global__ void __launch_bounds__(MtGeo<DK, DV>::NT, 1)
decode_mt_kernel(const DecodeArgs p, const int NH) {
    using Geo = MtGeo<DK, DV>;
    constexpr int RPL = Geo::RPL, NB = RPL == 2 ? 1 : RPL / 4, EPB = RPL == 2 ? 2 : 4;
    extern __shared__ __align__(128) unsigned char smem[];
    // T: the most tokens a sequence has in this launch (it sizes the shared buffers)
    const int T = p.T, W = p.sh.W, C = p.sh.C, Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk;
    const int TP = Geo::padded(T);  // token rows of the on-chip buffers
    const int npass = G / NH, NCH = 2 * DK + NH * DV;
    const int ngroups = p.B * Hk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* stage = reinterpret_cast<float*>(smem);
    uint16_t* rows = reinterpret_cast<uint16_t*>(smem + Geo::rows_off());
    uint16_t* wts = reinterpret_cast<uint16_t*>(smem + Geo::wts_off(W, T));
    float* qk = reinterpret_cast<float*>(smem + Geo::qk_off(W, T));
    float* vs = reinterpret_cast<float*>(smem + Geo::vs_off(W, T));
    float* os = vs;  // o_t of a column replaces v_t once the warp owning the column has read it
    uint16_t* zb = reinterpret_cast<uint16_t*>(smem + Geo::zb_off(W, T));
    TokenScalars* sc = reinterpret_cast<TokenScalars*>(smem + Geo::sc_off(W, T));
    float* gram = reinterpret_cast<float*>(smem + Geo::gram_off(W, T));
    float* coef = reinterpret_cast<float*>(smem + Geo::coef_off(W, T));
    float* dsm = reinterpret_cast<float*>(smem + Geo::dsm_off(W, T)) + warp * (kChunk * 16);
    volatile int* stage_slot = reinterpret_cast<volatile int*>(smem + Geo::ctl_off(W, T));
    volatile int* abort_flag = stage_slot + 1;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Geo::ctl_off(W, T) + 8);
    uint64_t* zbar = full + 1;
    volatile int* stage_tok0 = reinterpret_cast<volatile int*>(zbar + 1);  // the stage's first packed row
    volatile int* stage_ntok = stage_tok0 + 1;                             // and its token count

    auto item_group = [&](int u) { return (int)blockIdx.x + (u / npass) * (int)gridDim.x; };
    // Every thread: the copies of pass u into the stage (or, past the last pass,
    // nothing); `slot` is the pass's pool slot, `tok0` and `ntok` its sequence's first
    // packed row and token count, all read beforehand. The barrier expects one arrival
    // per thread (its asynchronous copies) and the tile bytes' arrival.
    auto prefetch = [&](int u, int slot, int tok0, int ntok) {
        const int group = item_group(u);
        if (group >= ngroups) return;
        const int seq = group / Hk, hk = group - seq * Hk, h0 = hk * G + (u % npass) * NH;
        const bool bad_slot = slot < 0 || slot >= p.P;
        const bool bad_len = ntok < 0 || ntok > T || (p.cu_seqlens && (tok0 < 0 || tok0 + ntok > p.total_rows));
        if (bad_slot || bad_len || ntok == 0) {  // skipped (flagged unless it simply has no tokens)
            if (tid == 0) {
                if (p.err_flag && bad_slot) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
                if (p.err_flag && bad_len) atomicOr(p.err_flag, GDN_DEVICE_ERR_SEQLEN_BIT);
                *stage_slot = -1;
                mbar_arrive(full);
            }
            mbar_arrive(full);
            return;
        }
        const int nrow = W - 1 + ntok;
        const int ch_q = hk * DK, ch_k = Hk * DK + hk * DK, ch_v = 2 * Hk * DK + h0 * DV;
        auto run_channel = [&](int lc) { return lc < DK ? ch_q + lc : (lc < 2 * DK ? ch_k + lc - DK : ch_v + lc - 2 * DK); };
        if (tid == 0) {
            *stage_slot = slot;
            *stage_tok0 = tok0;
            *stage_ntok = ntok;
            mbar_arrive_expect_tx(full, (uint32_t)(NH * Geo::TILE));
        }
        if (lane == 0) {  // the NH state tiles, contiguous in the pool: one bulk copy per warp (a
                          // warp issuing many serialises them)
            const char* tiles = reinterpret_cast<const char*>(p.state_pool + ((size_t)slot * Hv + h0) * (size_t)(DK * DV));
            const int tile_bytes = NH * Geo::TILE;
            for (int c = warp * kMtChunk; c < tile_bytes; c += Geo::NW * kMtChunk) {
                fence_proxy_async_smem();  // the stage's last reads (generic proxy) before the copies overwrite it
                tma_load_1d(smem + c, tiles + c, (uint32_t)min(kMtChunk, tile_bytes - c), full);
            }
        }
        // the W-1 history rows, then the T token rows, of the pass's channels; then the
        // channels' weights ([channel][W], three runs of consecutive channels; a 16-byte
        // group never straddles two runs since every run holds a multiple of 8 channels)
        const uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
        const uint16_t* x = p.qkv + (size_t)tok0 * C;
        const int nv = NCH / 8;
        for (int i = tid; i < nrow * nv; i += Geo::NT) {
            const int r = i / nv, lc = (i - r * nv) * 8, ch = run_channel(lc);
            cp_async_16(rows + r * NCH + lc, r < W - 1 ? hist + (size_t)r * C + ch : x + (size_t)(r - (W - 1)) * C + ch);
        }
        for (int i = tid; i < NCH * W / 8; i += Geo::NT) {
            const int lc = (i * 8) / W, off = i * 8 - lc * W;
            cp_async_16(wts + i * 8, p.conv_w + (size_t)run_channel(lc) * W + off);
        }
        cp_async_arrive(full);
    };
    // the first packed row and the token count of pass u's sequence
    auto tokens_of = [&](int u, int& tok0, int& ntok) {
        const int group = item_group(u);
        if (group >= ngroups) {
            tok0 = ntok = 0;
        } else if (p.cu_seqlens) {
            const int seq = group / Hk;
            tok0 = __ldg(p.cu_seqlens + seq);
            ntok = __ldg(p.cu_seqlens + seq + 1) - tok0;
        } else {
            tok0 = (group / Hk) * T;
            ntok = T;
        }
    };

    // the slot of pass u (-1 past the last pass)
    auto slot_of = [&](int u) {
        const int group = item_group(u);
        return group < ngroups ? __ldg(p.slots + group / Hk) : -1;
    };
    if (tid == 0) {
        mbar_init(full, Geo::NT + 1);  // every thread's copies, and the tile bytes
        mbar_init(zbar, Geo::NT);      // every thread's copies
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    // With programmatic dependent launch this grid may start while the previous one
    // drains (on the SMs its early finishers have left), so the first pass's state
    // tiles are prefetched into L2 now. The slot read here may be stale: it only steers
    // the hint, and L2 stays coherent with whatever that grid still writes. Nothing is
    // read for use before that grid has completed.
    if (warp == 0 && blockIdx.x < ngroups) {
        const int seq0 = (int)blockIdx.x / Hk, h00 = ((int)blockIdx.x - seq0 * Hk) * G;
        const int sl = __ldcg(p.slots + seq0);
        if (sl >= 0 && sl < p.P) {
            const char* t0 = reinterpret_cast<const char*>(p.state_pool + ((size_t)sl * Hv + h00) * (size_t)(DK * DV));
            for (int c = lane * kMtChunk; c < NH * Geo::TILE; c += 32 * kMtChunk)
                bulk_prefetch_l2(t0 + c, (uint32_t)min(kMtChunk, NH * Geo::TILE - c));
        }
    }
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    {
        int tok0 = 0, ntok = 0;
        tokens_of(0, tok0, ntok);
        prefetch(0, slot_of(0), tok0, ntok);
    }

    const int rg = lane >> 2, cg = lane & 3;
    const bool active = warp < Geo::NWH * NH;  // warps holding state columns in this launch's passes
    int zphase = 0;                            // z copies waited for so far
    const int hh = warp / Geo::NWH, col = 16 * (warp % Geo::NWH) + 4 * cg;
    for (int u = 0;; ++u) {
        const int group = item_group(u);
        if (group >= ngroups) break;
        const int pass = u % npass;
        const int seq = group / Hk, hk = group - seq * Hk, h0 = hk * G + pass * NH;
        bool ok = mbar_wait_deadline(full, (uint32_t)(u & 1), kWaitTimeoutNs, [&] { return *abort_flag != 0; });
        if (!__syncthreads_and(ok)) {
            if (tid == 0) {
                *abort_flag = 1;
                if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
                for (int i = 0; i < 1024; ++i) __nanosleep(64);  // copies in flight land before the CTA leaves
            }
            break;
        }
        const int slot = *stage_slot, tok0 = *stage_tok0, ntok = *stage_ntok;
        // the next pass's slot and tokens: loaded now, first used when the next copies
        // are issued
        const int next_slot = slot_of(u + 1);
        int next_tok0 = 0, next_ntok = 0;
        tokens_of(u + 1, next_tok0, next_ntok);
        if (slot < 0) {
            __syncthreads();  // every thread has read the stage's slot
            prefetch(u + 1, next_slot, next_tok0, next_ntok);
            continue;
        }
        {  // this pass's z rows (their buffer was last read before the barrier above)
            const int nv = NH * DV / 8;
            for (int i = tid; i < ntok * nv; i += Geo::NT) {
                const int t = i / nv, o = (i - t * nv) * 8;
                cp_async_16(zb + t * NH * DV + o, p.z + (((size_t)tok0 + t) * Hv + h0) * DV + o);
            }
            cp_async_arrive(zbar);
        }
        // the gate inputs of this pass's heads, loaded now and used after the conv
        uint16_t g_a = 0, g_b = 0;
        float g_A = 0.f, g_dt = 0.f;
        if (tid < ntok * NH) {
            const int t = tid / NH, k = tid - t * NH;
            const size_t ai = ((size_t)tok0 + t) * Hv + h0 + k;
            g_a = p.a[ai];
            g_b = p.b[ai];
            g_A = p.A_log[h0 + k];
            g_dt = p.dt_bias[h0 + k];
        }

        // ---- this warp's state columns into registers: P[pair][c] = (S[r][col+c], S[r+1][col+c])
        constexpr int NPR = RPL / 2;  // row pairs per lane
        f2 P[NPR][4];
        if (active) {
            const float* tile = stage + (size_t)hh * (DK * DV) + col;
#pragma unroll
            for (int j = 0; j < NB; ++j)
#pragma unroll
                for (int e = 0; e < EPB; e += 2) {
                    const float4 a = *reinterpret_cast<const float4*>(tile + mt_row<RPL>(j, rg, e) * DV);
                    const float4 b = *reinterpret_cast<const float4*>(tile + mt_row<RPL>(j, rg, e + 1) * DV);
                    f2* pr = P[(j * EPB + e) / 2];
                    pr[0] = f2_pack(a.x, b.x); pr[1] = f2_pack(a.y, b.y);
                    pr[2] = f2_pack(a.z, b.z); pr[3] = f2_pack(a.w, b.w);
                }
        }
        // ---- step 3: conv + SiLU of every channel for every token. A window of the last
        // K staged rows slides through registers with the newest row at the top, the
        // weights aligned to it (taps beyond W are zero), so every register index is a
        // compile-time constant: K = 4 when W = 4, else the widest conv supported.
        auto conv_channels = [&](auto taps) {
            constexpr int K = decltype(taps)::value;
            for (int lc = tid; lc < NCH; lc += Geo::NT) {
                float wr[K], win[K];
#pragma unroll
                for (int m = 0; m < K; ++m) {
                    const int j = W - K + m;  // tap of window position m: it multiplies staged row t + j
                    wr[m] = j >= 0 ? bf16_bits_to_float(wts[lc * W + j]) : 0.f;
                    // before token 0's shift position m holds staged row j - 1 (history rows only)
                    win[m] = j >= 1 ? bf16_bits_to_float(rows[(j - 1) * NCH + lc]) : 0.f;
                }
#pragma unroll 4
                for (int t = 0; t < ntok; ++t) {
#pragma unroll
                    for (int m = 0; m < K - 1; ++m) win[m] = win[m + 1];
                    win[K - 1] = bf16_bits_to_float(rows[(t + W - 1) * NCH + lc]);
                    float u2 = 0.f;
#pragma unroll
                    for (int m = 0; m < K; ++m) u2 = fmaf(wr[m], win[m], u2);
                    const float sv = silu_fast(u2);
                    if (lc < 2 * DK) {
                        qk[t * 2 * DK + lc] = sv;
                    } else {
                        const int v_h = (lc - 2 * DK) / DV, v_j = lc - 2 * DK - v_h * DV;
                        vs[(v_h * TP + t) * DV + v_j] = sv;
                    }
                }
            }
        };
        if (W == 4)
            conv_channels(Taps<4>{});
        else
            conv_channels(Taps<kMaxConvWidth>{});
        // ---- the new conv history: the last W-1 raw inputs. The v channels of this
        // pass's heads always; the k-head's q/k channels by the group's last pass.
        // A speculative verify writes no pool.
        const bool spec = p.spec_delta != nullptr;
        if (!spec) {
            uint16_t* hw = p.conv_pool + (size_t)slot * (W - 1) * C;
            const int lc0 = pass == npass - 1 ? 0 : 2 * DK, nvec = (NCH - lc0) / 8;
            const int ch_q = hk * DK, ch_k = Hk * DK + hk * DK, ch_v = 2 * Hk * DK + h0 * DV;
            for (int i = tid; i < (W - 1) * nvec; i += Geo::NT) {
                const int r = i / nvec, lc = lc0 + (i - r * nvec) * 8;
                const int ch = lc < DK ? ch_q + lc : (lc < 2 * DK ? ch_k + lc - DK : ch_v + lc - 2 * DK);
                *reinterpret_cast<uint4*>(hw + (size_t)r * C + ch) =
                    *reinterpret_cast<const uint4*>(rows + (ntok + r) * NCH + lc);
            }
        }
        // ---- steps 4, 5: decay and write strength per v-head and token. The tokens that pad
        // the last chunk get decay 1 and strength 0, and zero q, k and v: they change nothing.
        const int ntp = (ntok + kChunk - 1) / kChunk * kChunk;
        if (tid < ntp * NH) {
            const int t = tid / NH, k = tid - t * NH;
            TokenScalars& st = sc[t * Geo::NHC + k];
            if (t < ntok) {
                gate_and_beta(g_a, g_b, g_A, g_dt, st.alpha, st.beta);
            } else {
                st.alpha = 1.f;
                st.beta = 0.f;
            }
        }
        for (int i = tid; i < (ntp - ntok) * 2 * DK; i += Geo::NT) qk[ntok * 2 * DK + i] = 0.f;
        for (int i = tid; i < NH * (ntp - ntok) * DV; i += Geo::NT) {
            const int h = i / ((ntp - ntok) * DV), r = i - h * (ntp - ntok) * DV;
            vs[(h * TP + ntok) * DV + r] = 0.f;
        }
        __syncthreads();  // the stage is empty; k, q, v are in
        prefetch(u + 1, next_slot, next_tok0, next_ntok);
        // ---- step 3's L2 norms, as factors on the raw q and k, and the raw dot products
        // the chunked recurrence needs: a warp per token t, against the tokens of its chunk
        for (int t = warp; t < ntp; t += Geo::NW) {
            const int c0t = t - t % kChunk;
            const float* qt = qk + t * 2 * DK;
            const float* kt = qt + DK;
            float acc[kGramFloats - 3];  // k_i.k_t (4), k_i.q_t (4), q_t.q_t
#pragma unroll
            for (int i = 0; i < kGramFloats - 3; ++i) acc[i] = 0.f;
            for (int r = lane; r < DK; r += 32) {
                const float qv = qt[r], kv = kt[r];
#pragma unroll
                for (int i = 0; i < kChunk; ++i) {
                    const float ki = qk[(c0t + i) * 2 * DK + DK + r];
                    acc[i] = fmaf(ki, kv, acc[i]);
                    acc[kChunk + i] = fmaf(ki, qv, acc[kChunk + i]);
                }
                acc[2 * kChunk] = fmaf(qv, qv, acc[2 * kChunk]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int i = 0; i < kGramFloats - 3; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
            if (lane < kGramFloats - 3) {
                float v = acc[0];
#pragma unroll
                for (int i = 1; i < kGramFloats - 3; ++i) v = lane == i ? acc[i] : v;
                gram[t * kGramFloats + lane] = v;
            }
            const float nq = t < ntok ? rsqrtf(acc[2 * kChunk] + p.sh.l2_eps) * p.sh.q_scale : 0.f;
            float kk = acc[0];  // k_t . k_t
#pragma unroll
            for (int i = 1; i < kChunk; ++i) kk = t - c0t == i ? acc[i] : kk;
            const float nk = t < ntok ? rsqrtf(kk + p.sh.l2_eps) : 0.f;
            for (int k = lane; k < NH; k += 32) {
                TokenScalars& st = sc[t * Geo::NHC + k];
                st.nq = nq;
                st.nk = nk;
            }
        }
        __syncthreads();
        if (spec) {  // the verify call's factors: the normalised key (once per k-head) and the decays
            if (pass == npass - 1)
                for (int i = tid; i < ntok * DK; i += Geo::NT) {
                    const int t = i / DK, r = i - t * DK;
                    p.spec_k[(((size_t)tok0 + t) * Hk + hk) * DK + r] = qk[t * 2 * DK + DK + r] * sc[t * Geo::NHC].nk;
                }
            if (tid < ntok * NH) {
                const int t = tid / NH, k = tid - t * NH;
                p.spec_alpha[((size_t)tok0 + t) * Hv + h0 + k] = sc[t * Geo::NHC + k].alpha;
            }
        }
        // ---- the scalars of each (v-head, chunk). With the chunk's
        // decays a_j (j = 0..3), Gamma_j = a_0 ... a_j and A_ji = a_{i+1} ... a_j (A_jj = 1),
        // S0 = c0 S~ the state at the chunk's start and normalised k_j = nk_j k~_j,
        // q_j = nq_j q~_j (k~, q~ raw), the tokens of the chunk give
        //   delta_j = b_j v_j - b_j c0 Gamma_j nk_j (S~^T k~_j) - sum_{i<j} b_j A_ji (k_i.k_j) delta_i
        //   o_j     = c0 Gamma_j nq_j (S~^T q~_j) + sum_{i<=j} A_ji (k_i.q_j) delta_i
        //   S_end   = Gamma_3 S0 + sum_i A_3i k_i delta_i^T.
        // The registers keep S~ = S / c with c the running product of the decays; when c
        // would fall below 2^-64 it is folded into the registers (S~ <- c S~, c <- 1).
        // Block layout: b[4], ek[4] (on S~^T k~), eq[4] (on S~^T q~), L[6] (row j, i < j),
        // Q[10] (row j, i <= j), f[4] (factor of delta_i on k~_i in the update), the fold
        // multiplier, the fold flag and the running scale after the chunk.
        const int nchunk = ntp / kChunk;
        // A thread per coefficient: the running scale at its chunk's start (a scan over
        // the chunks before it), then the one entry.
        for (int e = tid; e < NH * nchunk * kCoefFloats; e += Geo::NT) {
            const int k = e / (nchunk * kCoefFloats), rem = e - k * nchunk * kCoefFloats;
            const int m = rem / kCoefFloats, idx = rem - m * kCoefFloats;
            const TokenScalars* sk = sc + k;  // token t of v-head k: sk[t * NHC]
            float c0 = 1.f;
            for (int mm = 0; mm < m; ++mm) {
                float gl = 1.f;
#pragma unroll
                for (int j = 0; j < kChunk; ++j) gl *= sk[(mm * kChunk + j) * Geo::NHC].alpha;
                const float cn = c0 * gl;
                c0 = cn < 0x1p-64f ? 1.f : cn;
            }
            const TokenScalars* s0 = sk + m * kChunk * Geo::NHC;
            auto al = [&](int j) { return s0[j * Geo::NHC].alpha; };
            auto gam = [&](int j) {  // decays of tokens 0..j of the chunk
                float r = 1.f;
                for (int x = 0; x <= j; ++x) r *= al(x);
                return r;
            };
            auto A = [&](int j, int i) {  // decays of tokens i+1..j of the chunk
                float r = 1.f;
                for (int x = i + 1; x <= j; ++x) r *= al(x);
                return r;
            };
            const float* gr = gram + m * kChunk * kGramFloats;  // row j: k_i.k_j (i < 4), k_i.q_j, q_j.q_j
            float v;
            if (idx < 4) {
                v = s0[idx * Geo::NHC].beta;
            } else if (idx < 8) {
                const int j = idx - 4;
                v = s0[j * Geo::NHC].beta * c0 * gam(j) * s0[j * Geo::NHC].nk;
            } else if (idx < 12) {
                const int j = idx - 8;
                v = c0 * gam(j) * s0[j * Geo::NHC].nq;
            } else if (idx < 18) {  // L, row j, i < j
                const int l = idx - 12, j = l < 1 ? 1 : (l < 3 ? 2 : 3), i = l - j * (j - 1) / 2;
                v = s0[j * Geo::NHC].beta * A(j, i) * s0[i * Geo::NHC].nk * s0[j * Geo::NHC].nk * gr[j * kGramFloats + i];
            } else if (idx < 28) {  // Q, row j, i <= j
                const int l = idx - 18, j = l < 1 ? 0 : (l < 3 ? 1 : (l < 6 ? 2 : 3)), i = l - j * (j + 1) / 2;
                v = A(j, i) * s0[i * Geo::NHC].nk * s0[j * Geo::NHC].nq * gr[j * kGramFloats + kChunk + i];
            } else {
                const float cn = c0 * gam(kChunk - 1);
                const bool fold = cn < 0x1p-64f;
                if (idx < 32) {
                    const int j = idx - 28;
                    v = fold ? A(kChunk - 1, j) * s0[j * Geo::NHC].nk : __fdividef(s0[j * Geo::NHC].nk, c0 * gam(j));
                } else if (idx == 32) {
                    v = fold ? cn : 1.f;
                } else if (idx == 33) {
                    v = fold ? 1.f : 0.f;
                } else if (idx == 34) {
                    v = fold ? 1.f : cn;
                } else {
                    v = 0.f;
                }
            }
            coef[(k * (TP / kChunk) + m) * kCoefFloats + idx] = v;
        }
        __syncthreads();

        // ---- steps 6, 7: the recurrence, a chunk of tokens at a time, on this warp's columns
        if (active) {
            float cfin = 1.f;  // the running scale after the last chunk
            for (int m = 0; m < nchunk; ++m) {
                const float* cf = coef + (hh * (TP / kChunk) + m) * kCoefFloats;
                const float* qk0 = qk + m * kChunk * 2 * DK;  // raw q then raw k of the chunk's tokens
                // S~^T k~_j for the chunk's tokens, two at a time, over this lane's rows (even and
                // odd rows apart), then summed over the row groups (lanes with the same columns)
                float mk[kChunk][4];
#pragma unroll
                for (int h2 = 0; h2 < kChunk; h2 += 2) {
                    f2 ak[2][4];
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) ak[j][cc] = 0ull;
#pragma unroll
                    for (int jb = 0; jb < NB; ++jb) {
                        const int r0 = mt_row<RPL>(jb, rg, 0);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float* kr = qk0 + (h2 + j) * 2 * DK + DK;
                            f2 kp[EPB / 2];
                            if constexpr (EPB == 4) {
                                const ulonglong2 k2 = *reinterpret_cast<const ulonglong2*>(kr + r0);
                                kp[0] = k2.x; kp[1] = k2.y;
                            } else {
                                kp[0] = *reinterpret_cast<const f2*>(kr + r0);
                            }
#pragma unroll
                            for (int e = 0; e < EPB / 2; ++e) {
                                const f2* pr = P[jb * (EPB / 2) + e];
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc) ak[j][cc] = f2_fma(pr[cc], kp[e], ak[j][cc]);
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const float2 x = f2_unpack(ak[j][cc]);
                            mk[h2 + j][cc] = x.x + x.y;
                        }
#pragma unroll
                    for (int off = Geo::CG; off < 32; off <<= 1)
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc)
                                mk[h2 + j][cc] += __shfl_xor_sync(0xffffffffu, mk[h2 + j][cc], off);
                }
                // delta of every token of the chunk (forward substitution), per column; the row
                // group 0 lanes keep it in this warp's shared buffer for the readout and update
                {
                    float d[kChunk][4];
                    int li = 12;
#pragma unroll
                    for (int j = 0; j < kChunk; ++j) {
                        const float4 v4 = *reinterpret_cast<const float4*>(vs + (hh * TP + m * kChunk + j) * DV + col);
                        const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
                        const float bj = cf[j], ekj = cf[4 + j];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) d[j][cc] = fmaf(-ekj, mk[j][cc], bj * vv[cc]);
#pragma unroll
                        for (int i = 0; i < j; ++i, ++li) {
                            const float l = cf[li];
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) d[j][cc] = fmaf(-l, d[i][cc], d[j][cc]);
                        }
                    }
                    if (rg == 0) {
#pragma unroll
                        for (int j = 0; j < kChunk; ++j) {
                            const float4 dj = make_float4(d[j][0], d[j][1], d[j][2], d[j][3]);
                            reinterpret_cast<float4*>(dsm + j * 16)[cg] = dj;
                            if (spec && m * kChunk + j < ntok)
                                *reinterpret_cast<float4*>(p.spec_delta +
                                                           (((size_t)tok0 + m * kChunk + j) * Hv + h0 + hh) * DV + col) = dj;
                        }
                    }
                }
                __syncwarp();  // every lane has read v of these columns before o replaces it, and delta is in
                auto delta = [&](int j) { return reinterpret_cast<const float4*>(dsm + j * 16)[cg]; };
                // S~^T q~_j two tokens at a time, then o_j
#pragma unroll
                for (int h2 = 0; h2 < kChunk; h2 += 2) {
                    f2 aq[2][4];
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) aq[j][cc] = 0ull;
#pragma unroll
                    for (int jb = 0; jb < NB; ++jb) {
                        const int r0 = mt_row<RPL>(jb, rg, 0);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float* qr = qk0 + (h2 + j) * 2 * DK;
                            f2 qp[EPB / 2];
                            if constexpr (EPB == 4) {
                                const ulonglong2 q2 = *reinterpret_cast<const ulonglong2*>(qr + r0);
                                qp[0] = q2.x; qp[1] = q2.y;
                            } else {
                                qp[0] = *reinterpret_cast<const f2*>(qr + r0);
                            }
#pragma unroll
                            for (int e = 0; e < EPB / 2; ++e) {
                                const f2* pr = P[jb * (EPB / 2) + e];
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc) aq[j][cc] = f2_fma(pr[cc], qp[e], aq[j][cc]);
                            }
                        }
                    }
                    float mq[2][4];
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const float2 x = f2_unpack(aq[j][cc]);
                            mq[j][cc] = x.x + x.y;
                        }
#pragma unroll
                    for (int off = Geo::CG; off < 32; off <<= 1)
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) mq[j][cc] += __shfl_xor_sync(0xffffffffu, mq[j][cc], off);
                    if (rg == 0) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int jj = h2 + j;
                            const int q0 = 18 + jj * (jj + 1) / 2;  // row jj of Q
                            float o[4];
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) o[cc] = cf[8 + jj] * mq[j][cc];
#pragma unroll
                            for (int i = 0; i <= jj; ++i) {
                                const float qc = cf[q0 + i];
                                const float4 di = delta(i);
                                o[0] = fmaf(qc, di.x, o[0]); o[1] = fmaf(qc, di.y, o[1]);
                                o[2] = fmaf(qc, di.z, o[2]); o[3] = fmaf(qc, di.w, o[3]);
                            }
                            *reinterpret_cast<float4*>(os + (hh * TP + m * kChunk + jj) * DV + col) =
                                make_float4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
                // the rank-4 update S~ <- s S~ + sum_j k~_j (f_j delta_j)^T (s = 1 unless the
                // running scale is folded in)
                if (cf[33] != 0.f) {
                    const f2 s2 = f2_pack(cf[32], cf[32]);
#pragma unroll
                    for (int i = 0; i < NPR; ++i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) P[i][cc] = f2_mul(P[i][cc], s2);
                }
#pragma unroll 1
                for (int j = 0; j < kChunk; ++j) {  // rolled: one token's k rows in flight at a time
                    const float fj = cf[28 + j];
                    const float* kr = qk0 + j * 2 * DK + DK;
                    const float4 dj = delta(j);
                    f2 dn[4];
                    dn[0] = f2_pack(dj.x * fj, dj.x * fj); dn[1] = f2_pack(dj.y * fj, dj.y * fj);
                    dn[2] = f2_pack(dj.z * fj, dj.z * fj); dn[3] = f2_pack(dj.w * fj, dj.w * fj);
#pragma unroll
                    for (int jb = 0; jb < NB; ++jb) {
                        const int r0 = mt_row<RPL>(jb, rg, 0);
                        f2 kp[EPB / 2];
                        if constexpr (EPB == 4) {
                            const ulonglong2 k2 = *reinterpret_cast<const ulonglong2*>(kr + r0);
                            kp[0] = k2.x; kp[1] = k2.y;
                        } else {
                            kp[0] = *reinterpret_cast<const f2*>(kr + r0);
                        }
#pragma unroll
                        for (int e = 0; e < EPB / 2; ++e) {
                            f2* pr = P[jb * (EPB / 2) + e];
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) pr[cc] = f2_fma(kp[e], dn[cc], pr[cc]);
                        }
                    }
                }
                cfin = cf[34];
            }
            const float c = cfin;
            // the state back to the pool, scale applied (streaming: nothing here reads it again)
            if (!spec) {
            float* Sg = p.state_pool + ((size_t)slot * Hv + h0 + hh) * (size_t)(DK * DV) + col;
#pragma unroll
            for (int j = 0; j < NB; ++j)
#pragma unroll
                for (int e = 0; e < EPB; e += 2) {
                    const f2* pr = P[(j * EPB + e) / 2];
                    const float2 x0 = f2_unpack(pr[0]), x1 = f2_unpack(pr[1]), x2 = f2_unpack(pr[2]), x3 = f2_unpack(pr[3]);
                    __stcs(reinterpret_cast<float4*>(Sg + (size_t)mt_row<RPL>(j, rg, e) * DV),
                           make_float4(x0.x * c, x1.x * c, x2.x * c, x3.x * c));
                    __stcs(reinterpret_cast<float4*>(Sg + (size_t)mt_row<RPL>(j, rg, e + 1) * DV),
                           make_float4(x0.y * c, x1.y * c, x2.y * c, x3.y * c));
                }
            }
        }
        __syncthreads();

        // ---- step 8 over each head, the norm weight and SiLU(z): a warp per (token, head),
        // four columns per lane (DV <= 128)
        const bool has_cols = 4 * lane < DV;
        const uint2 nw = has_cols ? __ldg(reinterpret_cast<const uint2*>(p.norm_w) + lane) : make_uint2(0u, 0u);
        if (!mbar_wait_deadline(zbar, (uint32_t)(zphase & 1), kWaitTimeoutNs, [&] { return *abort_flag != 0; })) {
            if (lane == 0) {
                *abort_flag = 1;
                if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
            }
        }
        ++zphase;
        for (int task = warp; task < ntok * NH; task += Geo::NW) {
            const int t = task / NH, k = task - t * NH;
            const float4 o = has_cols ? reinterpret_cast<const float4*>(os + (k * TP + t) * DV)[lane]
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (!has_cols) continue;
            const float inv = rsqrtf(ss / (float)DV + p.sh.rms_eps);
            const size_t base = (((size_t)tok0 + t) * Hv + h0 + k) * DV + 4 * lane;
            const uint2 zz = *reinterpret_cast<const uint2*>(zb + (t * NH + k) * DV + 4 * lane);
            const float y0 = o.x * inv * bf16_bits_to_float(nw.x & 0xffffu) * silu_fast(bf16_bits_to_float(zz.x & 0xffffu));
            const float y1 = o.y * inv * bf16_bits_to_float(nw.x >> 16) * silu_fast(bf16_bits_to_float(zz.x >> 16));
            const float y2 = o.z * inv * bf16_bits_to_float(nw.y & 0xffffu) * silu_fast(bf16_bits_to_float(zz.y & 0xffffu));
            const float y3 = o.w * inv * bf16_bits_to_float(nw.y >> 16) * silu_fast(bf16_bits_to_float(zz.y >> 16));
            uint2 packed;
            packed.x = (uint32_t)float_to_bf16_bits(y0) | ((uint32_t)float_to_bf16_bits(y1) << 16);
            packed.y = (uint32_t)float_to_bf16_bits(y2) | ((uint32_t)float_to_bf16_bits(y3) << 16);
            *reinterpret_cast<uint2*>(p.out + base) = packed;
            if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + base) = make_float4(y0, y1, y2, y3);
        }
    }
    if (*abort_flag && tid == 0) {  // a wait gave up: copies still in flight land before the CTA leaves
        for (int i = 0; i < 1024; ++i) __nanosleep(64);
    }
}

// The largest divisor of G that one pass can hold.
template <int DK, int DV>
int heads_per_pass(int G) {
    int nh = 1;
    for (int d = 1; d <= G && d <= MtGeo<DK, DV>::NHC; ++d)
        if (G % d == 0) nh = d;
    return nh;
}

// Per device and dynamic shared-memory size: the kernel attribute set, the SM count and
// the co-resident CTAs per SM, found once (eager callers pay no device queries per call).
struct MtLaunchInfo {
    int dev, smem, sms, per_sm;
};

template <int DK, int DV>
cudaError_t mt_launch_info(int smem, int* grid_cap) {
    static std::mutex mu;
    static std::vector<MtLaunchInfo> known;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const MtLaunchInfo& k : known)
        if (k.dev == dev && k.smem == smem) {
            *grid_cap = k.sms * k.per_sm;
            return cudaSuccess;
        }
    auto kern = decode_mt_kernel<DK, DV>;
    // the attribute is the largest size any launch on this device asks for
    int largest = smem;
    for (const MtLaunchInfo& k : known)
        if (k.dev == dev && k.smem > largest) largest = k.smem;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, largest)) != cudaSuccess)
        return e;
    int sms = 0, per_sm = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, MtGeo<DK, DV>::NT, smem)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    known.push_back({dev, smem, sms, per_sm});
    *grid_cap = sms * per_sm;
    return cudaSuccess;
}

template <int DK, int DV>
cudaError_t launch_mt(const DecodeArgs& a, cudaStream_t stream) {
    using Geo = MtGeo<DK, DV>;
    auto kern = decode_mt_kernel<DK, DV>;
    const int smem = Geo::total(a.sh.W, a.T);
    int cap = 0;
    cudaError_t e = mt_launch_info<DK, DV>(smem, &cap);
    if (e != cudaSuccess) return e;
    const int ngroups = a.B * a.sh.Hk;
    const int grid = ngroups < cap ? ngroups : cap;
    if (grid <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Geo::NT);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, heads_per_pass<DK, DV>(a.sh.Hv / a.sh.Hk));
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
