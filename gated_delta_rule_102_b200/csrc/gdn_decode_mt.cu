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
    // Shared memory (bytes, every block 16-byte aligned): the stage (NHC state tiles,
    // the staged raw rows and the weights), then the raw q and k per token, v per v-head
    // and token (replaced by o: the warp that reads v_t of a column writes o_t of it),
    // the z rows of the pass, the per-token scalars, the stage's slot and the abort
    // flag, and the stage and z barriers.
    static __host__ __device__ int rows_off() { return NHC * TILE; }
    static __host__ __device__ int wts_off(int W, int T) { return rows_off() + ((W - 1 + T) * NCHC * 2 + 15) / 16 * 16; }
    static __host__ __device__ int qk_off(int W, int T) { return wts_off(W, T) + (NCHC * W * 2 + 15) / 16 * 16; }
    static __host__ __device__ int vs_off(int W, int T) { return qk_off(W, T) + T * 2 * DK * 4; }
    static __host__ __device__ int zb_off(int W, int T) { return vs_off(W, T) + T * NHC * DV * 4; }
    static __host__ __device__ int sc_off(int W, int T) { return zb_off(W, T) + T * NHC * DV * 2; }
    static __host__ __device__ int ctl_off(int W, int T) {
        return (sc_off(W, T) + T * NHC * (int)sizeof(TokenScalars) + 15) / 16 * 16;
    }
    static __host__ __device__ int total(int W, int T) { return ctl_off(W, T) + 48; }
    // the control block: the stage's slot, the abort flag, the stage and z barriers,
    // the stage's first packed row and token count, and the stage and z phases a CTA
    // that gives up waits for before it leaves
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
    const int npass = G / NH, NCH = 2 * DK + NH * DV;
    const int ngroups_max = p.B * Hk;  // the launch's bound; the batch itself is read after the grid dependency
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float* stage = reinterpret_cast<float*>(smem);
    uint16_t* rows = reinterpret_cast<uint16_t*>(smem + Geo::rows_off());
    uint16_t* wts = reinterpret_cast<uint16_t*>(smem + Geo::wts_off(W, T));
    float* qk = reinterpret_cast<float*>(smem + Geo::qk_off(W, T));
    float* vs = reinterpret_cast<float*>(smem + Geo::vs_off(W, T));
    float* os = vs;  // o_t of a column replaces v_t once the warp owning the column has read it
    uint16_t* zb = reinterpret_cast<uint16_t*>(smem + Geo::zb_off(W, T));
    TokenScalars* sc = reinterpret_cast<TokenScalars*>(smem + Geo::sc_off(W, T));
    volatile int* stage_slot = reinterpret_cast<volatile int*>(smem + Geo::ctl_off(W, T));
    volatile int* abort_flag = stage_slot + 1;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Geo::ctl_off(W, T) + 8);
    uint64_t* zbar = full + 1;
    volatile int* stage_tok0 = reinterpret_cast<volatile int*>(zbar + 1);  // the stage's first packed row
    volatile int* stage_ntok = stage_tok0 + 1;                             // and its token count
    volatile int* drain = stage_ntok + 1;  // [2]: stage phase, z phase still in flight (-1: none)

    if (tid == 0) {
        mbar_init(full, Geo::NT + 1);  // every thread's copies, and the tile bytes
        mbar_init(zbar, Geo::NT);      // every thread's copies
        *abort_flag = 0;
        drain[0] = drain[1] = -1;
        mbar_init_fence();
    }
    __syncthreads();
    // With programmatic dependent launch this grid may start while the previous one
    // drains (on the SMs its early finishers have left), so the first pass's state
    // tiles are prefetched into L2 now. The slot read here may be stale: it only steers
    // the hint, and L2 stays coherent with whatever that grid still writes. Nothing is
    // read for use before that grid has completed.
    if (warp == 0 && blockIdx.x < ngroups_max) {
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
    const int ngroups = launch_batch(p.B_dev, p.B, p.err_flag, blockIdx.x == 0 && tid == 0) * Hk;

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
        bool ok = mbar_wait_deadline(full, (uint32_t)(u & 1), kWaitTimeoutCycles, [&] { return *abort_flag != 0; });
        if (!__syncthreads_and(ok)) {
            if (tid == 0) {
                *abort_flag = 1;
                drain[0] = u & 1;  // pass u's copies were issued and never waited for
                if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
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
                        vs[(v_h * T + t) * DV + v_j] = sv;
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
        // ---- steps 4, 5: decay and write strength per v-head and token
        if (tid < ntok * NH) {
            const int t = tid / NH, k = tid - t * NH;
            gate_and_beta(g_a, g_b, g_A, g_dt, sc[t * Geo::NHC + k].alpha, sc[t * Geo::NHC + k].beta);
        }
        __syncthreads();  // the stage is empty; k, q, v are in
        prefetch(u + 1, next_slot, next_tok0, next_ntok);
        // ---- L2 norms of q and k (step 3) as factors on the raw values, and k.q: a warp per token
        for (int t = warp; t < ntok; t += Geo::NW) {
            float sq = 0.f, sk = 0.f, dot = 0.f;
            for (int r = lane; r < DK; r += 32) {
                const float a = qk[t * 2 * DK + r], b = qk[t * 2 * DK + DK + r];
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
            const float nq = rsqrtf(sq + p.sh.l2_eps) * p.sh.q_scale, nk = rsqrtf(sk + p.sh.l2_eps);
            for (int k = lane; k < NH; k += 32) {
                TokenScalars& st = sc[t * Geo::NHC + k];
                st.nq = nq;
                st.nk = nk;
                st.kq = dot * nq * nk;
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

        // ---- steps 6, 7: the recurrence, token by token, on this warp's columns
        if (active) {
            float c = 1.f;  // S = c * S~ (the registers hold S~)
            for (int t = 0; t < ntok; ++t) {
                const float* qr = qk + t * 2 * DK;
                const float* kr = qr + DK;
                f2 ak[4], aq[4];  // per column: S~^T k and S~^T q over the even and the odd rows
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) ak[cc] = aq[cc] = 0ull;
#pragma unroll
                for (int j = 0; j < NB; ++j) {
                    const int r0 = mt_row<RPL>(j, rg, 0);
                    f2 kp[EPB / 2], qp[EPB / 2];  // (k_r, k_r+1) and (q_r, q_r+1) of this block's row pairs
                    if constexpr (EPB == 4) {
                        const ulonglong2 k2 = *reinterpret_cast<const ulonglong2*>(kr + r0);
                        const ulonglong2 q2 = *reinterpret_cast<const ulonglong2*>(qr + r0);
                        kp[0] = k2.x; kp[1] = k2.y; qp[0] = q2.x; qp[1] = q2.y;
                    } else {
                        kp[0] = *reinterpret_cast<const f2*>(kr + r0);
                        qp[0] = *reinterpret_cast<const f2*>(qr + r0);
                    }
#pragma unroll
                    for (int e = 0; e < EPB / 2; ++e) {
                        const f2* pr = P[j * (EPB / 2) + e];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            ak[cc] = f2_fma(pr[cc], kp[e], ak[cc]);
                            aq[cc] = f2_fma(pr[cc], qp[e], aq[cc]);
                        }
                    }
                }
                float mk[4], mq[4];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const float2 x = f2_unpack(ak[cc]), y = f2_unpack(aq[cc]);
                    mk[cc] = x.x + x.y;
                    mq[cc] = y.x + y.y;
                }
#pragma unroll
                for (int off = Geo::CG; off < 32; off <<= 1) {  // over the row groups (lanes with the same columns)
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        mk[cc] += __shfl_xor_sync(0xffffffffu, mk[cc], off);
                        mq[cc] += __shfl_xor_sync(0xffffffffu, mq[cc], off);
                    }
                }
                const TokenScalars st = sc[t * Geo::NHC + hh];
                const float4 v4 = *reinterpret_cast<const float4*>(vs + (hh * T + t) * DV + col);
                const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
                const float c1 = c * st.alpha;  // S after this token's decay is c1 * S~
                const float am = c1 * st.nk, aqs = c1 * st.nq;
                float d[4], o[4];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    d[cc] = st.beta * fmaf(-am, mk[cc], vv[cc]);
                    o[cc] = fmaf(aqs, mq[cc], d[cc] * st.kq);
                }
                if (spec && rg == 0)
                    *reinterpret_cast<float4*>(p.spec_delta + (((size_t)tok0 + t) * Hv + h0 + hh) * DV + col) =
                        make_float4(d[0], d[1], d[2], d[3]);
                __syncwarp();  // every lane has read v_t of these columns before o_t replaces it
                if (rg == 0) *reinterpret_cast<float4*>(os + (hh * T + t) * DV + col) = make_float4(o[0], o[1], o[2], o[3]);
                float f;  // the update's factor on the raw k: nk delta / c, with c the new scale
                if (c1 < 0x1p-64f) {  // fold the scale into the registers before it underflows
                    const f2 cc2 = f2_pack(c1, c1);
#pragma unroll
                    for (int i = 0; i < NPR; ++i)
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) P[i][cc] = f2_mul(P[i][cc], cc2);
                    c = 1.f;
                    f = st.nk;
                } else {
                    c = c1;
                    f = __fdividef(st.nk, c1);
                }
                f2 dn[4];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) dn[cc] = f2_pack(d[cc] * f, d[cc] * f);
                // S~ += k (nk delta / c)^T on this lane's rows
#pragma unroll
                for (int j = 0; j < NB; ++j) {
                    const int r0 = mt_row<RPL>(j, rg, 0);
                    f2 kp[EPB / 2];
                    if constexpr (EPB == 4) {
                        const ulonglong2 k2 = *reinterpret_cast<const ulonglong2*>(kr + r0);
                        kp[0] = k2.x; kp[1] = k2.y;
                    } else {
                        kp[0] = *reinterpret_cast<const f2*>(kr + r0);
                    }
#pragma unroll
                    for (int e = 0; e < EPB / 2; ++e) {
                        f2* pr = P[j * (EPB / 2) + e];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) pr[cc] = f2_fma(kp[e], dn[cc], pr[cc]);
                    }
                }
            }
            // the state back to the pool, scale applied (streaming: nothing here reads it again)
            float* Sg = p.state_pool + ((size_t)slot * Hv + h0 + hh) * (size_t)(DK * DV) + col;
#pragma unroll
            for (int j = 0; j < (spec ? 0 : NB); ++j)
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
        __syncthreads();

        // ---- step 8 over each head, the norm weight and SiLU(z): a warp per (token, head),
        // four columns per lane (DV <= 128)
        const bool has_cols = 4 * lane < DV;
        const uint2 nw = has_cols ? __ldg(reinterpret_cast<const uint2*>(p.norm_w) + lane) : make_uint2(0u, 0u);
        if (!mbar_wait_deadline(zbar, (uint32_t)(zphase & 1), kWaitTimeoutCycles, [&] { return *abort_flag != 0; })) {
            if (lane == 0) {
                *abort_flag = 1;
                drain[1] = zphase & 1;  // this pass's z copies were issued and never waited for
                if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
            }
        }
        ++zphase;
        for (int task = warp; task < ntok * NH; task += Geo::NW) {
            const int t = task / NH, k = task - t * NH;
            const float4 o = has_cols ? reinterpret_cast<const float4*>(os + (k * T + t) * DV)[lane]
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
    // A wait gave up: the copies this CTA still has in flight land (or a further bounded
    // wait runs out) before it leaves. Each barrier phase counts every copy issued into
    // it, and a phase is armed only once the one before it has been waited for, so at
    // most the phase whose wait gave up is outstanding on each barrier. (When the z wait
    // gives up first, the next pass's stage wait then gives up at once and records its
    // phase; a stage phase never armed is never recorded.)
    if (*abort_flag && tid == 0) {
        if (drain[0] >= 0) mbar_wait_bounded(full, (uint32_t)drain[0]);
        if (drain[1] >= 0) mbar_wait_bounded(zbar, (uint32_t)drain[1]);
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
    if (chunk_supported(a)) return launch_decode_chunk(a, stream);  // the tensor-core chunk form
    switch (a.sh.dk) {
        case 16: return mt_dispatch<16>(a, stream);
        case 32: return mt_dispatch<32>(a, stream);
        case 64: return mt_dispatch<64>(a, stream);
        case 128: return mt_dispatch<128>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace gdn
