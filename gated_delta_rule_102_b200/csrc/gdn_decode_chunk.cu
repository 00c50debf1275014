// Multi-token GDN decode step on the fifth-generation tensor cores, for dk = dv = 128:
// steps 3 to 8 and the SiLU(z) gate of steps 9+10+11 on the page
// "spark_model/forward/qwen3_5/linear_attention.rs", applied to the n <= 16 tokens of
// a launch as one chunk instead of one token after another.
//
// The chunk form. Per (sequence, v-head), with S0 the state before the launch, the
// normalised keys k_t and scaled queries q_t (t < n), gamma_t = alpha_0 ... alpha_t
// and g_ts = alpha_{s+1} ... alpha_t (products of the decays, never ratios: decays
// may underflow), unrolling the token-by-token update S_t = alpha_t S_{t-1} +
// k_t delta_t^T gives
//   delta_t = beta_t (v_t - gamma_t S0^T k_t) - sum_{s<t} beta_t g_ts (k_s.k_t) delta_s
//   o_t     = gamma_t S0^T q_t + sum_{s<=t} g_ts (q_t.k_s) delta_s
//   S_n     = gamma_{n-1} S0 + sum_s g_{n-1,s} k_s delta_s^T,
// exactly the single-token recurrence up to rounding order. S0^T [k | q] (128 x 128 by
// 128 x 32) and the rank-n update are dense contractions: they run as tcgen05.mma
// kind::tf32 with every operand split into a tf32 high part and the remainder
// (x = hi + lo exactly; hi*hi + hi*lo + lo*hi recovers fp32 accuracy, the dropped
// lo*lo term is ~2^-20 relative). The 16 x 16 triangular solve for delta runs on the
// CUDA cores, one thread per state column.
//
// Data. The transposed state S^T lives in TMEM (lane = column of S, i.e. a v
// channel; one fp32 per TMEM column), as high and low parts for the first GEMM and as
// gamma S0^T in the accumulator of the update; the new state leaves TMEM straight to
// the pool, each warp writing whole 128-byte rows. The state is read and written once
// per launch, so the step is bound by HBM like the single-token one.
//
// Roles (one CTA of 384 threads per SM, walking the (sequence, k-head) groups cid,
// cid + grid, ...; a group's G v-heads are its units):
//  * warps 4-11, the producers: per group the conv + SiLU of its q and k channels, the
//    L2 norms, the high/low operand tiles of [k | q] (K-major, 128-byte swizzle), k^T
//    and the Gram products k.k, q.k; per unit the conv of its v channels (two threads per
//    channel), the gates and the unit's solve coefficients, and the gated RMSNorm and
//    outputs of each solved unit; raw rows arrive by cp.async into shared memory, one
//    group or head ahead;
//  * warps 0-3, the consumers (thread c owns column c and TMEM lane c): state chunks
//    into TMEM, the two GEMMs (issued by threads 0 and 32), the state copies (issued by
//    thread 64: TMA bulk copies of 32 rows, 16 KiB, into a ring holding one tile), the
//    solve and the new state's stores.
// Groups and units pass from producers to consumers through double buffers guarded by
// mbarriers. Every wait is bounded by the SM cycle counter; on expiry the CTA sets the
// timeout bit, all roles leave their loops, and what was issued completes before the
// TMEM is freed and the CTA leaves.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <type_traits>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "gdn_tcgen05.cuh"

namespace gdn {
namespace {

constexpr int kCT = 16;   // tokens of one chunk: the most one launch holds per sequence
constexpr int kDK = 128, kDV = 128;
constexpr int kChunkRows = 32;                       // state rows per ring buffer
constexpr int kChunkBytes = kChunkRows * kDV * 4;    // 16 KiB
constexpr int kChunksPerTile = kDK / kChunkRows;     // 4
constexpr int kRing = 4;                             // ring buffers: one state tile in flight
constexpr int kConsumerWarps = 4, kProducerWarps = 8;
constexpr int kProducers = 32 * kProducerWarps;
constexpr int kThreads = 32 * (kConsumerWarps + kProducerWarps);
constexpr int kConsumerBar = 1, kProducerBar = 2;    // named barriers (consumers, producers)

// [k_0..k_15 | q_0..q_15] x dk as the B operand of S0^T [k|q]^T: the tf32 high parts in
// rows 0..31 and the low parts in rows 32..63, K = dk, K-major with the 128-byte swizzle,
// one 8 KiB region (64 rows x 128 bytes) per 32 dk.
constexpr int kXRegion = 64 * 128;
constexpr int kXBuf = (kDK / 32) * kXRegion;   // 32 KiB
// k^T as the B operand of the update (N = dk rows, K = tokens): row r holds the high parts
// of k_0..k_15 [r] in its first 64 bytes and the low parts in the next 64, K-major with
// the 128-byte swizzle (an MN-major tf32 operand would need another swizzle atom).
constexpr int kZBuf = kDK * 128;                 // 16 KiB
constexpr int kScrStride = 2 * kDK + 4;          // producer scratch row: raw q, raw k, pad
constexpr int kRawRows = kMaxConvWidth - 1 + kCT;  // staged conv input rows: history, then tokens
// per group (producers only): the q and k channels' raw rows [kRawRows][256] and weights [256][W]
constexpr int kGroupRawBytes = kRawRows * 2 * kDK * 2 + 2 * kDK * kMaxConvWidth * 2;
// per unit (producers only, in the scratch's place): the v channels' raw rows and weights
constexpr int kUnitRawBytes = kRawRows * kDV * 2 + kDV * kMaxConvWidth * 2;
// per unit (double-buffered): v [16][128] f32 (replaced by o once the consumers have solved),
// alpha, beta, gamma, w [16], the solve's coefficients A [16][16] and M [16][16], z [16][128]
// bf16, and the unit's first packed row, v-head and token count (ints)
constexpr int kHeadFloats = kCT * kDV + 4 * kCT + 2 * kCT * kCT + kCT * kDV / 2 + 4;

// shared-memory byte offsets from a 1024-byte aligned base
constexpr int OFF_RING = 0;
constexpr int OFF_X = OFF_RING + kRing * kChunkBytes;
constexpr int OFF_Z = OFF_X + 2 * kXBuf;
constexpr int OFF_GRAM = OFF_Z + 2 * kZBuf;              // [2][k.k 256 | q.k 256] f32
constexpr int OFF_SCR = OFF_GRAM + 2 * 2 * kCT * kCT * 4;
constexpr int OFF_GRAW = OFF_SCR + kCT * kScrStride * 4;
constexpr int OFF_NRM = OFF_GRAW + kGroupRawBytes;       // [16] q factors, [16] k factors
constexpr int OFF_HEAD = OFF_NRM + 2 * kCT * 4;
constexpr int OFF_BAR = OFF_HEAD + 2 * kHeadFloats * 4;
// ring full [kRing], group full/empty [2] each, unit full/empty [2] each, the update's
// MMAs, the first GEMM's MMAs (two issuing threads)
constexpr int kNumBars = kRing + 8 + 2;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;  // TMEM address, abort flag, first-GEMM commits
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;  // + alignment slack
static_assert(OFF_X % 1024 == 0 && OFF_Z % 1024 == 0 && kXRegion % 1024 == 0, "swizzled operand alignment");
static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
static_assert(kUnitRawBytes <= kCT * kScrStride * 4 && OFF_GRAW % 16 == 0 && OFF_HEAD % 16 == 0, "staging");
static_assert(kSmemBytes <= 232448, "shared memory");

// TMEM columns (one fp32 per column per lane)
constexpr uint32_t TM_AHI = 0, TM_ALO = 128;  // S0^T high and low parts (K = dk)
constexpr uint32_t TM_D2 = 256;               // the update's accumulator: S_n^T
constexpr uint32_t TM_D1 = 384;   // S0_hi^T [k | q]_hi^T and S0_hi^T [k | q]_lo^T: 2 x 32 columns
constexpr uint32_t TM_D1B = 448;  // S0_lo^T [k | q]_hi^T: 32 columns (issued by another thread)
constexpr uint32_t TM_YHI = 480, TM_YLO = 496;  // A of the update: g_{n-1,t} delta_t (K = 16 tokens)
constexpr uint32_t kTmemCols = 512;
static_assert(TM_YLO + kCT <= kTmemCols, "TMEM columns");

__device__ __forceinline__ uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xFFFFE000u; }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// all of this thread's committed copy groups but the newest have landed
__device__ __forceinline__ void cp_async_wait_all_but_newest() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// conv + SiLU of one channel from its staged inputs: rows[r * stride] for r < W-1 the
// history, then the n <= 16 tokens; w: its W <= KW weights. out[t] for t < n, 0 beyond.
// KW is the width the code is unrolled for (taps past W are zero).
template <int KW>
__device__ __forceinline__ void conv_staged(const uint16_t* rows, int stride, const uint16_t* w, int W, int n,
                                            float (&out)[kCT]) {
    float xs[kCT + KW - 1];  // xs[KW - 1 + i] = input i (i < 0: history)
#pragma unroll
    for (int i = -(KW - 1); i < kCT; ++i) {
        const bool in = i < 0 ? -i <= W - 1 : i < n;
        xs[KW - 1 + i] = in ? bf16_bits_to_float(rows[(W - 1 + i) * stride]) : 0.f;
    }
    float wt[KW];  // wt[d] multiplies the input d tokens back
#pragma unroll
    for (int d = 0; d < KW; ++d) wt[d] = d < W ? bf16_bits_to_float(w[W - 1 - d]) : 0.f;
#pragma unroll
    for (int t = 0; t < kCT; ++t) {
        float u = 0.f;
#pragma unroll
        for (int d = KW - 1; d >= 0; --d) u = fmaf(wt[d], xs[KW - 1 + t - d], u);
        out[t] = t < n ? silu_fast(u) : 0.f;
    }
}

// The same for the NT tokens t0 .. t0 + NT - 1 only (inputs t0 - (KW - 1) .. t0 + NT - 1).
template <int KW, int NT>
__device__ __forceinline__ void conv_staged_run(const uint16_t* rows, int stride, const uint16_t* w, int W, int n,
                                                int t0, float (&out)[NT]) {
    float xs[NT + KW - 1];  // xs[KW - 1 + j] = input t0 + j (negative: history)
#pragma unroll
    for (int j = -(KW - 1); j < NT; ++j) {
        const int ii = t0 + j;
        const bool in = ii < 0 ? -ii <= W - 1 : ii < n;
        xs[KW - 1 + j] = in ? bf16_bits_to_float(rows[(W - 1 + ii) * stride]) : 0.f;
    }
    float wt[KW];
#pragma unroll
    for (int d = 0; d < KW; ++d) wt[d] = d < W ? bf16_bits_to_float(w[W - 1 - d]) : 0.f;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        float u = 0.f;
#pragma unroll
        for (int d = KW - 1; d >= 0; --d) u = fmaf(wt[d], xs[KW - 1 + t - d], u);
        out[t] = t0 + t < n ? silu_fast(u) : 0.f;
    }
}

// KW: the conv width the producers' convs are unrolled for, 4 (conv widths up to 4) or
// kMaxConvWidth: the shorter unrolling halves the conv's instructions and the kernel's code,
// and the producers' conv phases are bound by issue, not by memory.
template <int KW>
__global__ void __launch_bounds__(kThreads, 1) decode_chunk_kernel(const DecodeArgs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, W = p.sh.W, Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk;
    const size_t C = (size_t)p.sh.C;
    const bool spec = p.spec_delta != nullptr;  // verify: no pool is written
    float* ring = reinterpret_cast<float*>(smem + OFF_RING);
    unsigned char* xbuf = smem + OFF_X;
    unsigned char* zbuf = smem + OFF_Z;
    float* gram = reinterpret_cast<float*>(smem + OFF_GRAM);
    float* scr = reinterpret_cast<float*>(smem + OFF_SCR);
    uint16_t* uraw = reinterpret_cast<uint16_t*>(smem + OFF_SCR);  // (the unit phase's staging)
    uint16_t* graw = reinterpret_cast<uint16_t*>(smem + OFF_GRAW);
    float* nrm = reinterpret_cast<float*>(smem + OFF_NRM);
    float* heads = reinterpret_cast<float*>(smem + OFF_HEAD);
    uint64_t* ring_full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* grp_full = ring_full + kRing;
    uint64_t* grp_empty = grp_full + 2;
    uint64_t* unit_full = grp_empty + 2;
    uint64_t* unit_empty = unit_full + 2;
    uint64_t* mma_bar = unit_empty + 2;  // the update GEMM (thread 0)
    uint64_t* g1_bar = mma_bar + 1;      // the first GEMM (threads 0 and 32)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    uint32_t* g1_commits = tmem_slot + 2;  // first-GEMM batches thread 0 has committed (for an abort)

    if (tid == 0) {
        for (int s = 0; s < kRing; ++s) mbar_init(ring_full + s, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(grp_full + b, kProducerWarps);
            mbar_init(grp_empty + b, kConsumerWarps);
            mbar_init(unit_full + b, kProducerWarps);
            mbar_init(unit_empty + b, kConsumerWarps);
        }
        mbar_init(mma_bar, 1);
        mbar_init(g1_bar, 2);
        *abort_flag = 0;
        *g1_commits = 0;
        mbar_init_fence();
    }
    if (warp == 0) tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the inputs may be written by the kernel before this one in the stream
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int ngroups = launch_batch(p.B_dev, p.B, p.err_flag, blockIdx.x == 0 && tid == 0) * Hk;

    auto fail = [&]() {
        *abort_flag = 1;
        if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait_deadline(bar, parity, kWaitTimeoutCycles, [&] { return *abort_flag != 0; });
    };
    // Group g's slot, first packed row and token count. Every role evaluates it the
    // same way and skips the same groups (a bad slot or token count, or no tokens).
    auto group_info = [&](int g, int& slot, int& tok0, int& n, bool& bad_slot, bool& bad_len) {
        const int seq = g / Hk;
        slot = __ldg(p.slots + seq);
        if (p.cu_seqlens) {
            tok0 = __ldg(p.cu_seqlens + seq);
            n = __ldg(p.cu_seqlens + seq + 1) - tok0;
        } else {
            tok0 = seq * T;
            n = T;
        }
        bad_slot = slot < 0 || slot >= p.P;
        bad_len = n < 0 || n > T || (p.cu_seqlens && (tok0 < 0 || tok0 + n > p.total_rows));
        return !bad_slot && !bad_len && n > 0;
    };
    // The same, split in two: the loads of a group's slot and offsets (issued one group ahead,
    // so their latency passes while the group before runs), then the decision.
    struct GroupRaw {
        int slot, tok0, end;
    };
    auto group_fetch = [&](int g) {
        GroupRaw r{-1, 0, 0};
        if (g >= ngroups) return r;
        const int seq = g / Hk;
        r.slot = __ldg(p.slots + seq);
        if (p.cu_seqlens) {
            r.tok0 = __ldg(p.cu_seqlens + seq);
            r.end = __ldg(p.cu_seqlens + seq + 1);
        } else {
            r.tok0 = seq * T;
            r.end = r.tok0 + T;
        }
        return r;
    };
    auto group_eval = [&](const GroupRaw& r, int& slot, int& tok0, int& n, bool& bad_slot, bool& bad_len) {
        slot = r.slot;
        tok0 = r.tok0;
        n = r.end - r.tok0;
        bad_slot = slot < 0 || slot >= p.P;
        bad_len = n < 0 || n > T || (p.cu_seqlens && (tok0 < 0 || tok0 + n > p.total_rows));
        return !bad_slot && !bad_len && n > 0;
    };

    if (warp >= kConsumerWarps) {
        // ---- producers: thread i handles conv channel i of the group's q | k (256) and, for
        // i < 128, channel i of each unit's v; the group's bad slots and token counts are
        // flagged here
        const int i = tid - 32 * kConsumerWarps, pw = warp - kConsumerWarps;
        int li = 0, hu = 0;  // groups and units produced
        int gstaged = -1;    // the group whose q/k rows and weights are in (or on their way to) graw
        int emitted = -1;    // the last unit whose outputs are written
        // cp.async of group gg's q and k channels: their history and token rows (16-byte
        // pieces, two runs of 128 channels per row) and weights (two runs of 128 W)
        auto stage_group = [&](int gg, int sl, int t0, int nn) {
            const int kh = gg % Hk, nr = W - 1 + nn;
            const uint16_t* hs = p.conv_pool + (size_t)sl * (W - 1) * C;
            const uint16_t* xs = p.qkv + (size_t)t0 * C;
            for (int e = i; e < nr * 32; e += kProducers) {
                const int r = e >> 5, part = (e >> 4) & 1, off = (e & 15) * 8;
                const size_t ch = (size_t)(part * Hk + kh) * kDK + off;
                cp_async_16(graw + r * 2 * kDK + part * kDK + off,
                            r < W - 1 ? hs + (size_t)r * C + ch : xs + (size_t)(r - (W - 1)) * C + ch);
            }
            const int wpieces = kDK * W / 8;
            uint16_t* gwt = graw + kRawRows * 2 * kDK;
            for (int e = i; e < 2 * wpieces; e += kProducers) {
                const int part = e >= wpieces, o = e - part * wpieces;
                cp_async_16(gwt + part * kDK * W + o * 8, p.conv_w + (size_t)(part * Hk + kh) * kDK * W + o * 8);
            }
            cp_async_commit();
            gstaged = gg;
        };
        // the RMSNorm weights of this lane's four columns (the same for every unit)
        const uint2 nw4 = __ldg(reinterpret_cast<const uint2*>(p.norm_w) + lane);
        const float nw[4] = {bf16_bits_to_float(nw4.x & 0xffffu), bf16_bits_to_float(nw4.x >> 16),
                             bf16_bits_to_float(nw4.y & 0xffffu), bf16_bits_to_float(nw4.y >> 16)};
        // step 8 and the SiLU(z) gate of a solved unit in buffer ub: a warp per token, four
        // columns per lane
        auto emit_unit = [&](int ub) {
            const float* ov = heads + ub * kHeadFloats;
            const uint16_t* oz = reinterpret_cast<const uint16_t*>(ov + kCT * kDV + 4 * kCT + 2 * kCT * kCT);
            const int* meta = reinterpret_cast<const int*>(ov + kHeadFloats - 4);
            const int ut0 = meta[0], uh = meta[1], un = meta[2];
            for (int t = pw; t < un; t += kProducerWarps) {
                const float4 o4 = reinterpret_cast<const float4*>(ov + t * kDV)[lane];
                float ss = o4.x * o4.x + o4.y * o4.y + o4.z * o4.z + o4.w * o4.w;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float inv = rsqrtf(ss * (1.0f / (float)kDV) + p.sh.rms_eps);
                const uint2 z2 = reinterpret_cast<const uint2*>(oz + t * kDV)[lane];
                const float y0 = o4.x * inv * nw[0] * silu_fast(bf16_bits_to_float(z2.x & 0xffffu));
                const float y1 = o4.y * inv * nw[1] * silu_fast(bf16_bits_to_float(z2.x >> 16));
                const float y2 = o4.z * inv * nw[2] * silu_fast(bf16_bits_to_float(z2.y & 0xffffu));
                const float y3 = o4.w * inv * nw[3] * silu_fast(bf16_bits_to_float(z2.y >> 16));
                const size_t oi = (((size_t)ut0 + t) * Hv + uh) * kDV + 4 * lane;
                uint2 packed;
                packed.x = (uint32_t)float_to_bf16_bits(y0) | ((uint32_t)float_to_bf16_bits(y1) << 16);
                packed.y = (uint32_t)float_to_bf16_bits(y2) | ((uint32_t)float_to_bf16_bits(y3) << 16);
                *reinterpret_cast<uint2*>(p.out + oi) = packed;
                if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + oi) = make_float4(y0, y1, y2, y3);
            }
        };
        GroupRaw cur = group_fetch(blockIdx.x), nxt;
        int gn = 0;
        for (int g = blockIdx.x; g < ngroups; g = gn, cur = nxt) {
            gn = g + (int)gridDim.x;
            nxt = group_fetch(gn);  // used by the next iteration
            int slot, tok0, n;
            bool bad_slot, bad_len;
            const bool run = group_eval(cur, slot, tok0, n, bad_slot, bad_len);
            if (i == 0 && p.err_flag && bad_slot) atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
            if (i == 0 && p.err_flag && bad_len) atomicOr(p.err_flag, GDN_DEVICE_ERR_SEQLEN_BIT);
            if (!run) continue;
            const int gb = li & 1, hk = g % Hk;
            bool ok = li < 2 || wait(grp_empty + gb, (uint32_t)(((li >> 1) - 1) & 1));
            // (also: this group's scratch is free, every producer having read the last one)
            if (!named_barrier_and(kProducerBar, kProducers, ok && !*abort_flag)) {
                if (!ok) fail();
                break;
            }
            uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
            const uint16_t* x = p.qkv + (size_t)tok0 * C;
            const int nrow = W - 1 + n;
            uint16_t* gw = graw + kRawRows * 2 * kDK;  // weights [256][W]
            if (gstaged != g) stage_group(g, slot, tok0, n);  // (normally staged while the group before ran)
            cp_async_wait_all();
            named_barrier(kProducerBar, kProducers);
            {  // step 3 for channel i of q | k: conv + SiLU into the scratch
                float qk[kCT];
                const int lc = i, part = i / kDK;
                conv_staged<KW>(graw + lc, 2 * kDK, gw + lc * W, W, n, qk);
#pragma unroll
                for (int t = 0; t < kCT; ++t) scr[t * kScrStride + lc] = qk[t];
                if (!spec)  // the new history: the last W-1 raw inputs
                    for (int r = 0; r < W - 1; ++r)
                        hist[(size_t)r * C + (size_t)(part * Hk + hk) * kDK + (i - part * kDK)] =
                            graw[(n + r) * 2 * kDK + lc];
            }
            named_barrier(kProducerBar, kProducers);
            {  // the staging buffer is free: the rows of the next group this CTA runs (normally the one
               // fetched ahead, whose slot and offsets have arrived during the conv)
                int g2 = gn, s2 = 0, t2 = 0, n2 = 0;
                bool b2s, b2l;
                if (g2 < ngroups && !group_eval(nxt, s2, t2, n2, b2s, b2l))
                    for (g2 += (int)gridDim.x; g2 < ngroups && !group_info(g2, s2, t2, n2, b2s, b2l);)
                        g2 += (int)gridDim.x;
                if (g2 < ngroups) stage_group(g2, s2, t2, n2);
            }
            // L2 norms of q and k per token (step 3): factors on the raw values
#pragma unroll
            for (int m = 0; m < kCT / kProducerWarps; ++m) {  // a warp per token
                const int t = pw + kProducerWarps * m;
                float sq = 0.f, sk = 0.f;
#pragma unroll
                for (int r = lane; r < kDK; r += 32) {
                    const float a = scr[t * kScrStride + r], b = scr[t * kScrStride + kDK + r];
                    sq = fmaf(a, a, sq);
                    sk = fmaf(b, b, sk);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                if (lane == 0) {
                    nrm[t] = rsqrtf(sq + p.sh.l2_eps) * p.sh.q_scale;
                    nrm[kCT + t] = rsqrtf(sk + p.sh.l2_eps);
                }
            }
            named_barrier(kProducerBar, kProducers);
            {  // the operand tiles: row r < 16 the normalised k_r, row 16 + t the scaled q_t
                const int row = i >> 3;
                const bool isk = row < kCT;
                const int t = isk ? row : row - kCT;
                const float f = isk ? nrm[kCT + t] : nrm[t];
                const float* src = scr + t * kScrStride + (isk ? kDK : 0);
                unsigned char* xh = xbuf + gb * kXBuf;  // high parts in rows 0..31, low in 32..63
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int j = (i & 7) + 8 * m;  // 16-byte group: dk 4j .. 4j+3
                    float4 v = *reinterpret_cast<const float4*>(src + 4 * j);
                    v.x *= f; v.y *= f; v.z *= f; v.w *= f;
                    const uint4 h = make_uint4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
                    const uint4 l = make_uint4(__float_as_uint(v.x - __uint_as_float(h.x)),
                                               __float_as_uint(v.y - __uint_as_float(h.y)),
                                               __float_as_uint(v.z - __uint_as_float(h.z)),
                                               __float_as_uint(v.w - __uint_as_float(h.w)));
                    const int off = (j >> 3) * kXRegion + row * 128 + (((j & 7) ^ (row & 7)) << 4);
                    *reinterpret_cast<uint4*>(xh + off) = h;
                    *reinterpret_cast<uint4*>(xh + off + 32 * 128) = l;
                    if (spec && isk && t < n)
                        *reinterpret_cast<float4*>(p.spec_k + (((size_t)tok0 + t) * Hk + hk) * kDK + 4 * j) = v;
                }
            }
            {  // k^T for the update: row r = dk index, high then low parts of k_0..k_15 [r]; thread
               // i takes row i % 128 and the token quads 2 (i / 128) and 2 (i / 128) + 1
                const int zrow = i & (kDK - 1);
                unsigned char* zr = zbuf + gb * kZBuf + zrow * 128;
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int j = 2 * (i / kDK) + jj;
                    float kx[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        kx[e] = scr[(4 * j + e) * kScrStride + kDK + zrow] * nrm[kCT + 4 * j + e];
                    const uint4 h = make_uint4(tf32_hi(kx[0]), tf32_hi(kx[1]), tf32_hi(kx[2]), tf32_hi(kx[3]));
                    const uint4 l = make_uint4(__float_as_uint(kx[0] - __uint_as_float(h.x)),
                                               __float_as_uint(kx[1] - __uint_as_float(h.y)),
                                               __float_as_uint(kx[2] - __uint_as_float(h.z)),
                                               __float_as_uint(kx[3] - __uint_as_float(h.w)));
                    *reinterpret_cast<uint4*>(zr + ((j ^ (zrow & 7)) << 4)) = h;
                    *reinterpret_cast<uint4*>(zr + (((j + 4) ^ (zrow & 7)) << 4)) = l;
                }
            }
            {  // Gram products of the normalised vectors: k_t.k_s and q_t.k_s, thread i one (t, s)
                const int t = i >> 4, s0 = i & 15;
                const float* qt = scr + t * kScrStride;
                const float* kt = qt + kDK;
                const float* k0 = scr + s0 * kScrStride + kDK;
                float4 kk4 = make_float4(0.f, 0.f, 0.f, 0.f), qk4 = kk4;  // four independent chains each
#pragma unroll 8
                for (int r = 0; r < kDK; r += 4) {
                    const float4 a = *reinterpret_cast<const float4*>(kt + r);
                    const float4 b = *reinterpret_cast<const float4*>(qt + r);
                    const float4 c0 = *reinterpret_cast<const float4*>(k0 + r);
                    kk4.x = fmaf(a.x, c0.x, kk4.x); kk4.y = fmaf(a.y, c0.y, kk4.y);
                    kk4.z = fmaf(a.z, c0.z, kk4.z); kk4.w = fmaf(a.w, c0.w, kk4.w);
                    qk4.x = fmaf(b.x, c0.x, qk4.x); qk4.y = fmaf(b.y, c0.y, qk4.y);
                    qk4.z = fmaf(b.z, c0.z, qk4.z); qk4.w = fmaf(b.w, c0.w, qk4.w);
                }
                const float kk0 = (kk4.x + kk4.y) + (kk4.z + kk4.w), qk0 = (qk4.x + qk4.y) + (qk4.z + qk4.w);
                float* gr = gram + gb * 2 * kCT * kCT;
                gr[t * kCT + s0] = kk0 * nrm[kCT + t] * nrm[kCT + s0];
                gr[kCT * kCT + t * kCT + s0] = qk0 * nrm[t] * nrm[kCT + s0];
            }
            fence_proxy_async_smem();  // the operand tiles are read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(grp_full + gb);
            ++li;

            // ---- the group's units (v-heads)
            const float* KK = gram + gb * 2 * kCT * kCT;
            const float* QK = KK + kCT * kCT;
            bool stop = false;
            const int gi = i - (kProducers - 32);  // the last producer warp's lanes 0..15: the gates of token gi
            // cp.async of head hh's v channel rows and weights into the staging area (free once every
            // producer has passed the group's Gram products, or the last head's v conv)
            uint16_t* uw = uraw + kRawRows * kDV;  // weights [128][W]
            auto stage_v = [&](int hh) {
                const size_t cv = (size_t)2 * Hk * kDK + (size_t)hh * kDV;
                for (int e = i; e < nrow * 16; e += kProducers) {
                    const int r = e >> 4, off = (e & 15) * 8;
                    cp_async_16(uraw + r * kDV + off, r < W - 1 ? hist + (size_t)r * C + cv + off
                                                            : x + (size_t)(r - (W - 1)) * C + cv + off);
                }
                for (int e = i; e < kDV * W / 8; e += kProducers) cp_async_16(uw + e * 8, p.conv_w + cv * W + e * 8);
                cp_async_commit();
            };
            // cp.async of head hh's z rows into unit buffer ub (free once its last unit is emitted)
            auto stage_z = [&](int hh, int ub) {
                uint16_t* zb2 =
                    reinterpret_cast<uint16_t*>(heads + ub * kHeadFloats + kCT * kDV + 4 * kCT + 2 * kCT * kCT);
                for (int e = i; e < n * 16; e += kProducers) {
                    const int t = e >> 4, off = (e & 15) * 8;
                    cp_async_16(zb2 + t * kDV + off, p.z + (((size_t)tok0 + t) * Hv + hh) * kDV + off);
                }
                cp_async_commit();
            };
            // the gate inputs of head hh's tokens and its gate parameters (loaded one head ahead
            // within the group, so that no load is outstanding at the barrier after the gates)
            uint16_t ga = 0, gbb = 0;
            float gA = 0.f, gdt = 0.f;
            auto load_gates = [&](int hh) {
                if (gi >= 0 && gi < kCT && gi < n) {
                    const size_t ai = ((size_t)tok0 + gi) * Hv + hh;
                    ga = p.a[ai];
                    gbb = p.b[ai];
                    gA = __ldg(p.A_log + hh);
                    gdt = __ldg(p.dt_bias + hh);
                }
            };
            for (int j = 0; j < G; ++j, ++hu) {
                const int hb = hu & 1, h = hk * G + j;
                ok = hu < 2 || wait(unit_empty + hb, (uint32_t)(((hu >> 1) - 1) & 1));
                if (!named_barrier_and(kProducerBar, kProducers, ok && !*abort_flag)) {
                    if (!ok) fail();
                    stop = true;
                    break;
                }
                if (j == 0) {  // the group's first head: its v rows and gate inputs travel under the emit
                    stage_v(h);
                    load_gates(h);
                }
                if (hu >= 2 && emitted < hu - 2) {  // the unit solved two units ago leaves the buffer first
                    emit_unit(hb);
                    emitted = hu - 2;
                    named_barrier(kProducerBar, kProducers);
                }
                float* hv = heads + hb * kHeadFloats;  // v [16][128]
                float* ha = hv + kCT * kDV;            // alpha [16], beta, gamma, w, A [16][16], M [16][16]
                float* hbeta = ha + kCT;
                float* hgam = hbeta + kCT;
                float* hw = hgam + kCT;
                float* hA = hw + kCT;
                float* hM = hA + kCT * kCT;
                if (i == 0) {
                    int* meta = reinterpret_cast<int*>(hv + kHeadFloats - 4);
                    meta[0] = tok0;
                    meta[1] = h;
                    meta[2] = n;
                }
                const size_t chv = (size_t)2 * Hk * kDK + (size_t)h * kDV;
                if (j == 0) stage_z(h, hb);  // (later heads' z rows were staged while the one before ran)
                // this head's v rows have landed; its z rows, the newest copies, may still be on their
                // way: they are read only by the emit, after another wait of this kind or the drain's
                cp_async_wait_all_but_newest();
                named_barrier(kProducerBar, kProducers);
                if (gi >= 0 && gi < kCT) {  // steps 4, 5 per token (no decay and no write past the tokens)
                    float al = 1.f, be = 0.f;
                    if (gi < n) {
                        gate_and_beta(ga, gbb, gA, gdt, al, be);
                        if (spec) p.spec_alpha[((size_t)tok0 + gi) * Hv + h] = al;
                    }
                    ha[gi] = al;
                    hbeta[gi] = be;
                }
                {  // step 3 for v channel i % 128 of this head, tokens 8 (i / 128) .. 8 (i / 128) + 7
                    constexpr int kHalf = kCT / 2;
                    const int vc = i & (kDV - 1), t0 = (i / kDV) * kHalf;
                    float vv[kHalf];
                    conv_staged_run<KW, kHalf>(uraw + vc, kDV, uw + vc * W, W, n, t0, vv);
#pragma unroll
                    for (int t = 0; t < kHalf; ++t) hv[(t0 + t) * kDV + vc] = vv[t];
                    if (!spec && t0 == 0)
                        for (int r = 0; r < W - 1; ++r) hist[(size_t)r * C + chv + vc] = uraw[(n + r) * kDV + vc];
                }
                named_barrier(kProducerBar, kProducers);
                if (j + 1 < G) {  // the staging area is free: the next head's v rows and gate inputs
                    stage_v(h + 1);
                    load_gates(h + 1);
                }
                // the solve's coefficients: A_ts = beta_t g_ts k_t.k_s (s < t), M_ts = g_ts q_t.k_s (s <= t)
                {  // the decays in registers: every product below is a chain of selects and multiplies
                    float al[kCT];
#pragma unroll
                    for (int b4 = 0; b4 < kCT / 4; ++b4) {
                        const float4 a4 = reinterpret_cast<const float4*>(ha)[b4];
                        al[4 * b4] = a4.x; al[4 * b4 + 1] = a4.y; al[4 * b4 + 2] = a4.z; al[4 * b4 + 3] = a4.w;
                    }
                    const int e = i, t = e >> 4, s = e & 15;  // one coefficient pair per thread
                    float gts = 1.f;                           // alpha_{s+1} .. alpha_t
#pragma unroll
                    for (int u = 1; u < kCT; ++u) gts *= (u > s && u <= t) ? al[u] : 1.f;
                    hA[e] = s < t ? hbeta[t] * gts * KK[e] : 0.f;
                    hM[e] = s <= t ? gts * QK[e] : 0.f;
                    if (i < kCT) {  // gamma_t = alpha_0..alpha_t; w_s = alpha_{s+1}..alpha_{n-1}
                        float gm = 1.f, w = 1.f;
#pragma unroll
                        for (int u = 0; u < kCT; ++u) {
                            gm *= u <= i ? al[u] : 1.f;
                            w *= (u > i && u < n) ? al[u] : 1.f;
                        }
                        hgam[i] = gm;
                        hw[i] = i < n ? w : 0.f;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(unit_full + hb);
                if (j + 1 < G) {  // the next head's buffer: its previous unit leaves, its z rows start
                    const int nb = (hu + 1) & 1;
                    const bool ok2 = hu < 1 || wait(unit_empty + nb, (uint32_t)(((hu - 1) >> 1) & 1));
                    if (!named_barrier_and(kProducerBar, kProducers, ok2 && !*abort_flag)) {
                        if (!ok2) fail();
                        stop = true;
                        break;
                    }
                    if (hu >= 1 && emitted < hu - 1) {
                        emit_unit(nb);
                        emitted = hu - 1;
                    }
                    named_barrier(kProducerBar, kProducers);  // the buffer's z rows are read
                    stage_z(h + 1, nb);
                }
            }
            if (stop) break;
        }
        // the last two units' outputs (every producer takes the same decision; their z rows have
        // landed before the barrier)
        cp_async_wait_all();
        if (named_barrier_and(kProducerBar, kProducers, !*abort_flag))
            for (int u = emitted + 1; u < hu; ++u) {
                const bool got = wait(unit_empty + (u & 1), (uint32_t)((u >> 1) & 1));
                if (!named_barrier_and(kProducerBar, kProducers, got && !*abort_flag)) {
                    if (!got) fail();
                    break;
                }
                emit_unit(u & 1);
            }
        cp_async_wait_all();  // no copy of this thread lands after the CTA has left
    } else {
        // ---- consumers: thread c owns state column c (TMEM lane c). A wait that gives
        // up is agreed on at the next consumer barrier, where all four warps leave
        // together; tcgen05 loads and stores are never under a lane-divergent branch.
        // A unit's new state leaves TMEM while the next unit's tile goes in: chunk q of
        // the accumulator is stored just before the next unit's chunk q overwrites it.
        const int c = tid;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        int li = 0, hu = 0, chunk = 0;
        uint32_t mma_issued = 0, mma_seen = 0;  // update commits issued (counted by all) and waited for (own)
        uint32_t g1_seen = 0;                   // first-GEMM phases waited for (own)
        float* pend = nullptr;                  // column c of the state tile still in the accumulator
        bool ok = true;
        auto store_chunk = [&](int q) {         // rows 32q .. 32q+31 of the pending tile
            float col[32];
            tmem_ld32(lane_base + TM_D2 + 32 * q, col);
#pragma unroll
            for (int r = 0; r < 32; ++r) __stcs(pend + (size_t)(32 * q + r) * kDV, col[r]);
        };
        // Thread 64 issues the state copies: the ring holds one tile (kRing = 4 chunks), and
        // a unit's chunk q is copied into buffer q as soon as the unit before it has taken
        // its own chunk q into TMEM (after that chunk's consumer barrier).
        static_assert(kRing == kChunksPerTile, "one tile in the ring");
        constexpr size_t kTileElems = (size_t)kDK * kDV;
        constexpr int kCopier = 64;        // the thread (warp 2) that issues the state copies
        int issued = 0;                    // chunks the copier has armed
        const float* next_tile = nullptr;  // the state tile of the unit after the current one
        auto next_group = [&](int from, int& sl) {  // the first group >= from this CTA runs
            int gg = from, t0, nn;
            bool bs, bl;
            while (gg < ngroups && !group_info(gg, sl, t0, nn, bs, bl)) gg += (int)gridDim.x;
            return gg;
        };
        auto issue_chunk = [&](const float* tile, int q) {
            fence_proxy_async_smem();  // the buffer's last reads (generic proxy) before the copy
            mbar_arrive_expect_tx(ring_full + q, (uint32_t)kChunkBytes);
            tma_load_1d(ring + (size_t)q * (kChunkBytes / 4), tile + (size_t)q * kChunkRows * kDV,
                        (uint32_t)kChunkBytes, ring_full + q);
            ++issued;
        };
        if (c == kCopier) {
            int sl = 0;
            const int g0 = next_group(blockIdx.x, sl);
            if (g0 < ngroups)
                for (int q = 0; q < kChunksPerTile; ++q)
                    issue_chunk(p.state_pool + ((size_t)sl * Hv + (g0 % Hk) * G) * kTileElems, q);
        }
        GroupRaw cur = group_fetch(blockIdx.x), nxt;
        int gn = 0;
        for (int g = blockIdx.x; g < ngroups; g = gn, cur = nxt) {
            gn = g + (int)gridDim.x;
            nxt = group_fetch(gn);  // used by the next iteration
            int slot, tok0, n;
            bool bad_slot, bad_len;
            if (!group_eval(cur, slot, tok0, n, bad_slot, bad_len)) continue;
            const int gb = li & 1, hk = g % Hk;
            const bool got = wait(grp_full + gb, (uint32_t)((li >> 1) & 1));
            if (!named_barrier_and(kConsumerBar, 128, got && !*abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t xb = smem_addr(xbuf + gb * kXBuf);
            const uint32_t zb = smem_addr(zbuf + gb * kZBuf);
            for (int j = 0; j < G; ++j, ++hu) {
                const int hb = hu & 1, h = hk * G + j;
                float* hv = heads + hb * kHeadFloats;  // v, then o
                const float* ha = hv + kCT * kDV;
                const float* hbeta = ha + kCT;
                const float* hgam = hbeta + kCT;
                const float* hw = hgam + kCT;
                const float* hA = hw + kCT;
                const float* hM = hA + kCT * kCT;
                if (c == kCopier) {
                    int sl2 = slot, g2 = g;
                    if (j + 1 >= G) {  // the next group: normally the one fetched ahead
                        int t2, n2;
                        bool b2s, b2l;
                        g2 = gn;
                        if (g2 < ngroups && !group_eval(nxt, sl2, t2, n2, b2s, b2l)) g2 = next_group(gn + (int)gridDim.x, sl2);
                    }
                    next_tile = g2 < ngroups
                                    ? p.state_pool + ((size_t)sl2 * Hv + (g2 % Hk) * G + (g2 == g ? j + 1 : 0)) * kTileElems
                                    : nullptr;
                }
                bool w = wait(unit_full + hb, (uint32_t)((hu >> 1) & 1));
                const float gC = hgam[n - 1];
                // ---- the state tile into TMEM chunk by chunk (S0^T high and low parts, and
                // gamma_{n-1} S0^T in the accumulator); after each chunk's barrier the next
                // unit's chunk q is copied into the buffer just read
                for (int q = 0; q < kChunksPerTile; ++q, ++chunk) {
                    const int s = chunk % kRing;
                    w = w && wait(ring_full + s, (uint32_t)((chunk / kRing) & 1));
                    if (pend) store_chunk(q);
                    const float* src = ring + (size_t)s * (kChunkBytes / 4) + c;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {  // 16 rows at a time
                        uint32_t hi[16], lo[16], dd[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) {
                            const float x = src[(16 * hh + r) * kDV];
                            hi[r] = tf32_hi(x);
                            lo[r] = __float_as_uint(x - __uint_as_float(hi[r]));
                            dd[r] = __float_as_uint(gC * x);
                        }
                        const uint32_t col = 32 * q + 16 * hh;
                        tmem_st16(lane_base + TM_AHI + col, hi);
                        tmem_st16(lane_base + TM_ALO + col, lo);
                        if (!spec) tmem_st16(lane_base + TM_D2 + col, dd);
                    }
                    w = __all_sync(0xffffffffu, w);
                    tmem_wait_st();
                    tcgen05_fence_before();
                    if (!named_barrier_and(kConsumerBar, 128, w && !*abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (c == kCopier && next_tile) issue_chunk(next_tile, q);  // every consumer has read buffer q
                }
                if (!ok) break;
                // the first GEMM, S0^T [k | q]^T, once the whole tile is in (the consumers' barriers
                // are not held up by its issue): the high part of S0 against the high and low operand
                // tiles side by side (N = 64) from thread 0, its low part against the high tiles
                // (N = 32) from thread 32, each into its own accumulator (a fixed order per
                // accumulator); K = 8 per MMA
                if (c == 0 || c == 32) {
                    tcgen05_fence_after();
#pragma unroll 1
                    for (int q = 0; q < kChunksPerTile; ++q) {
                        const uint64_t bx = sw128_desc(xb + q * kXRegion);
                        if (c == 0) {
                            constexpr uint32_t idesc64 = idesc_tf32(4 * kCT, 0);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_tf32_ts(tmem + TM_D1, tmem + TM_AHI + 32 * q + 8 * kk, bx + (uint64_t)(2 * kk),
                                             idesc64, (q | kk) != 0 ? 1u : 0u);
                        } else {
                            constexpr uint32_t idesc32 = idesc_tf32(2 * kCT, 0);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_tf32_ts(tmem + TM_D1B, tmem + TM_ALO + 32 * q + 8 * kk, bx + (uint64_t)(2 * kk),
                                             idesc32, (q | kk) != 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(smem_addr(g1_bar));
                    if (c == 0) ++*g1_commits;
                }
                pend = nullptr;
                float vv[kCT];
#pragma unroll
                for (int t = 0; t < kCT; ++t) vv[t] = hv[t * kDV + c];
                w = wait(g1_bar, g1_seen & 1u);
                if (w) ++g1_seen;
                tcgen05_fence_after();
                float d1[32];  // [S0^T k_t]_c for t < 16, then [S0^T q_t]_c: the three partial sums added
#pragma unroll
                for (int part = 0; part < 6; ++part) {  // 16 columns of one partial sum at a time
                    float pa[16];
                    const int h16 = part & 1, which = part >> 1;
                    tmem_ld16(lane_base + (which == 0 ? TM_D1 : which == 1 ? TM_D1 + 32 : TM_D1B) + 16 * h16, pa);
#pragma unroll
                    for (int j2 = 0; j2 < 16; ++j2) d1[16 * h16 + j2] = which == 0 ? pa[j2] : d1[16 * h16 + j2] + pa[j2];
                }
                // ---- steps 6, 7: the triangular solve for delta and the outputs, column c
                // (the coefficients of token t read as one row of float4s)
                float dl[kCT], o[kCT];
                float4 be4 = make_float4(0.f, 0.f, 0.f, 0.f), gm4 = be4;
#pragma unroll
                for (int t = 0; t < kCT; ++t) {
                    if ((t & 3) == 0) {
                        be4 = reinterpret_cast<const float4*>(hbeta)[t >> 2];
                        gm4 = reinterpret_cast<const float4*>(hgam)[t >> 2];
                    }
                    const float bet = (t & 3) == 0 ? be4.x : (t & 3) == 1 ? be4.y : (t & 3) == 2 ? be4.z : be4.w;
                    const float gmt = (t & 3) == 0 ? gm4.x : (t & 3) == 1 ? gm4.y : (t & 3) == 2 ? gm4.z : gm4.w;
                    float av[kCT], mv[kCT];
#pragma unroll
                    for (int b4 = 0; b4 <= t / 4; ++b4) {
                        const float4 x0 = reinterpret_cast<const float4*>(hA + t * kCT)[b4];
                        const float4 x1 = reinterpret_cast<const float4*>(hM + t * kCT)[b4];
                        av[4 * b4] = x0.x; av[4 * b4 + 1] = x0.y; av[4 * b4 + 2] = x0.z; av[4 * b4 + 3] = x0.w;
                        mv[4 * b4] = x1.x; mv[4 * b4 + 1] = x1.y; mv[4 * b4 + 2] = x1.z; mv[4 * b4 + 3] = x1.w;
                    }
                    float xd = bet * fmaf(-gmt, d1[t], vv[t]);
                    float xo = gmt * d1[kCT + t];
#pragma unroll
                    for (int s = 0; s < t; ++s) {
                        xd = fmaf(-av[s], dl[s], xd);
                        xo = fmaf(mv[s], dl[s], xo);
                    }
                    dl[t] = t < n ? xd : 0.f;
                    o[t] = fmaf(mv[t], dl[t], xo);
                }
                // o of column c replaces v_c (this thread has read it) for the producers'
                // gated RMSNorm
#pragma unroll
                for (int t = 0; t < kCT; ++t) hv[t * kDV + c] = o[t];
                if (spec) {
#pragma unroll
                    for (int t = 0; t < kCT; ++t)
                        if (t < n) p.spec_delta[(((size_t)tok0 + t) * Hv + h) * kDV + c] = dl[t];
                } else {  // A of the update: w_t delta_t, high and low parts
                    uint32_t yh[kCT], yl[kCT];
#pragma unroll
                    for (int t = 0; t < kCT; ++t) {
                        const float y = hw[t] * dl[t];
                        yh[t] = tf32_hi(y);
                        yl[t] = __float_as_uint(y - __uint_as_float(yh[t]));
                    }
                    tmem_st16(lane_base + TM_YHI, yh);
                    tmem_st16(lane_base + TM_YLO, yl);
                    tmem_wait_st();
                }
                tcgen05_fence_before();
                if (!named_barrier_and(kConsumerBar, 128, w && !*abort_flag)) {
                    ok = false;
                    break;
                }
                if (!spec) {
                    if (c == 0) {  // S_n^T = gamma S0^T + (w delta)^T k, B = k^T (K = tokens)
                        tcgen05_fence_after();
                        constexpr uint32_t idesc = idesc_tf32(kDK, 0);
                        const uint64_t bz = sw128_desc(zb);
#pragma unroll
                        for (int kk = 0; kk < kCT / 8; ++kk) {  // 8 tokens per MMA; low parts of k at 64 bytes
                            umma_tf32_ts(tmem + TM_D2, tmem + TM_YHI + 8 * kk, bz + (uint64_t)(2 * kk), idesc, 1u);
                            umma_tf32_ts(tmem + TM_D2, tmem + TM_YHI + 8 * kk, bz + (uint64_t)(2 * (kk + 2)), idesc, 1u);
                            umma_tf32_ts(tmem + TM_D2, tmem + TM_YLO + 8 * kk, bz + (uint64_t)(2 * kk), idesc, 1u);
                        }
                        umma_commit(smem_addr(mma_bar));
                    }
                    ++mma_issued;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(unit_empty + hb);  // inputs consumed, o written
                if (!spec) {  // the update is done: the tile is stored during the next unit's chunks
                    w = wait(mma_bar, mma_seen & 1u);
                    if (w) ++mma_seen;
                    tcgen05_fence_after();
                    pend = p.state_pool + ((size_t)slot * Hv + h) * (size_t)(kDK * kDV) + c;
                }
                tcgen05_fence_before();
                if (!named_barrier_and(kConsumerBar, 128, w && !*abort_flag)) {
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(grp_empty + gb);  // the group's operand tiles are free
            ++li;
        }
        if (ok && pend) {  // the last unit's tile
            tcgen05_fence_after();
            for (int q = 0; q < kChunksPerTile; ++q) store_chunk(q);
        }
        if (!ok) {
            fail();
            // an MMA batch of either GEMM that was issued and never waited for completes before
            // TMEM is freed, and the state copies still in flight land before the CTA leaves
            if (c == 0 && *g1_commits > g1_seen) mbar_wait_bounded(g1_bar, g1_seen & 1u);
            if (c == 0 && mma_issued > mma_seen) mbar_wait_bounded(mma_bar, mma_seen & 1u);
            if (c == kCopier)
                for (int v = chunk; v < issued; ++v) mbar_wait_bounded(ring_full + v % kRing, (uint32_t)((v / kRing) & 1));
        }
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Per device: the kernel attribute set and the SM count, found once.
cudaError_t chunk_grid_cap(int* cap) {
    static std::mutex mu;
    static int sms_of[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (sms_of[dev] == 0) {
        if ((e = cudaFuncSetAttribute(decode_chunk_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmemBytes)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(decode_chunk_kernel<kMaxConvWidth>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmemBytes)) != cudaSuccess)
            return e;
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_chunk_kernel<kMaxConvWidth>, kThreads, kSmemBytes)) !=
            cudaSuccess)
            return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        sms_of[dev] = sms;  // one CTA per SM: it holds all of TMEM
    }
    *cap = sms_of[dev];
    return cudaSuccess;
}

}  // namespace

// Every multi-token launch at dk = dv = 128, ragged ones included: a sequence without
// tokens costs nothing, one with fewer than 16 costs a whole tile like one with 16, and still
// the chunk form measured ahead of the register kernel on 64 sequences of 0..16 tokens (108
// against 119 us).
bool chunk_supported(const DecodeArgs& a) {
    return a.sh.dk == kDK && a.sh.dv == kDV && a.T >= 1 && a.T <= kCT && a.sh.W >= 1 &&
           a.sh.W <= kMaxConvWidth && a.sh.Hk >= 1 && a.sh.Hv % a.sh.Hk == 0;
}

cudaError_t launch_decode_chunk(const DecodeArgs& a, cudaStream_t stream) {
    int cap = 0;
    cudaError_t e = chunk_grid_cap(&cap);
    if (e != cudaSuccess) return e;
    const long ngroups = (long)a.B * a.sh.Hk;
    const int grid = ngroups < cap ? (int)ngroups : cap;
    if (grid <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return a.sh.W <= 4 ? cudaLaunchKernelEx(&cfg, decode_chunk_kernel<4>, a)
                       : cudaLaunchKernelEx(&cfg, decode_chunk_kernel<kMaxConvWidth>, a);
}

}  // namespace gdn
