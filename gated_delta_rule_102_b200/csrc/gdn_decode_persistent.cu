// Persistent, warp-specialised form of the fused GDN decode step for single-token
// launches over many sequences (steps 3 to 8 and the SiLU(z) gate of steps 9+10+11
// on the page "spark_model/forward/qwen3_5/linear_attention.rs").
//
// Work. A cluster of G = Hv/Hk CTAs (one per v-head sharing a k-head) stays resident
// and walks (sequence, k-head) groups cid, cid + ncl, cid + 2 ncl, ... Each CTA owns
// one v-head of every group it visits: the whole dk x dv fp32 state tile of that
// head, contiguous in the pool.
//
// Roles inside a CTA.
//  * Warp 0, the loader, only issues TMA bulk copies: as soon as stage v % NSTAGE is
//    free it starts the copies of unit v's state tile and z row (completing on the
//    stage's `full` barrier) and of its conv inputs (history rows, x, weights) and
//    a/b values (completing on `cbar`).
//  * Warps 1-4, the finishers, take units in order once their conv inputs have
//    landed: they convolve this CTA's channels (its share of the k-head's q/k
//    channels plus its v-head's v channels), send the raw q/k share to every CTA of
//    the cluster with st.async (completed on the receiver's mbarrier) and roll the
//    conv history. The first finisher warp then waits for the other shares, tells
//    the consumers that q/k and v are in (the stage's `full` barrier), and
//    publishes the q/k norms, k.q and the gates on the stage's `pub` barrier.
//  * The remaining eight warps form two teams that take units in turn. A team owns
//    a unit: each warp holds a band of columns (the columns of S are independent
//    under the update), reads the tile from shared memory for S^T k and S^T q and
//    reduces over dk with shuffles, then (once `pub` has completed) reads it again
//    for the update and streams the new rows straight to the pool; each warp frees
//    its part of the stage after that, and the team applies the RMSNorm, the norm
//    weight and SiLU(z).
// Every channel's conv history is therefore read and rolled by exactly one CTA, the
// state is read once and written once, and HBM sees a steady stream of TMA loads and
// row stores instead of alternating load, compute and store phases.
//
// Every wait is an mbarrier poll bounded by the SM cycle counter. When one expires the
// CTA sets the timeout bit of the error flag, all roles leave their loops, the loader
// waits (bounded) for the copies of the stages it armed, and the CTA leaves through the
// final cluster barrier.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kTileChunk = 16384;  // bytes per bulk copy of a state tile
constexpr int kMaxConvWidthPersistent = 4;

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }
__host__ __device__ constexpr int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

struct StageInfo {  // what the producer publishes for a staged unit
    float alpha, beta, nq, nk, kq;
    int slot;   // -1: the unit's slot is out of range
    int group;  // (sequence, k-head) group of the unit; kEndOfWork: no more units
    int pad;
};
constexpr int kEndOfWork = -1;
constexpr int kRing = 16;  // group indices relayed from the cluster's rank 0 (dynamic schedule)
// Units 0 .. kFixedUnits - 1 of every CTA are groups cid + u * ncl under either
// schedule; their state tiles are prefetched into L2 before the grid dependency wait.
constexpr int kFixedUnits = 2;
static_assert(kFixedUnits >= 1 && kFixedUnits <= 8, "fixed units: four prefetch lanes each");

template <int DK, int DV>
struct WS {
    static constexpr int CONSUMER_WARPS = 8;
    static constexpr int FINISHER_WARPS = 4;
    static constexpr int PRODUCER_WARPS = 1 + FINISHER_WARPS;  // the copy-issuing warp, then the conv/gate warps
    static constexpr int NT = 32 * (PRODUCER_WARPS + CONSUMER_WARPS);
    static constexpr int MAX_HV = 128;        // A_log, dt_bias held in shared memory
    static constexpr int TEAM_WARPS = DV >= 128 ? 4 : (DV >= 64 ? 2 : 1);
    static constexpr int NTEAMS = CONSUMER_WARPS / TEAM_WARPS;
    static constexpr int CPW = DV / TEAM_WARPS;  // columns per consumer warp (32, or 16 when dv = 16)
    static constexpr int CG = CPW / 4;           // float4 column groups per warp
    static constexpr int RG = 32 / CG;           // row groups per warp
    static constexpr int RPL = DK / RG;          // rows per lane
    static constexpr int TILE_BYTES = DK * DV * 4;
    static constexpr int MAXNCH = 2 * DK + DV;   // most conv channels one CTA owns (G = 1)
    // staged conv inputs of one unit: W rows (W-1 history rows, then x) of the CTA's
    // channels, then the channels' W weights
    static constexpr int CROWS = kMaxConvWidthPersistent * MAXNCH * 2;
    static constexpr int CSTAGE = round_up(CROWS, 16) + round_up(MAXNCH * kMaxConvWidthPersistent * 2, 16);
    // as many stages as fit: each costs its tile, conv inputs, z, v, info and a q/k buffer
    static constexpr int PER_STAGE = TILE_BYTES + CSTAGE + DV * 6 + 32 + 2 * DK * 4 + 24 + 32;
    static constexpr int NSTAGE = clampi((232448 - 3072 - 4 * DK * 4) / PER_STAGE, 2, 8);
    static constexpr int QB = NSTAGE + 2;        // q/k buffers: two more than stages (see the finishers)
    // shared-memory byte offsets
    static constexpr int TILES = 0;
    static constexpr int CONV = TILES + NSTAGE * TILE_BYTES;        // [NSTAGE] staged conv inputs
    static constexpr int AB = CONV + NSTAGE * CSTAGE;               // [NSTAGE][2][8] bf16: a, b groups
    static constexpr int GP = AB + NSTAGE * 32;                     // [2][MAX_HV] f32: A_log, dt_bias
    static constexpr int ZB = GP + 2 * MAX_HV * 4;                  // [NSTAGE][DV] bf16
    static constexpr int VS = ZB + round_up(NSTAGE * DV * 2, 16);    // [NSTAGE][DV] f32
    static constexpr int SI = VS + NSTAGE * DV * 4;                  // [NSTAGE] StageInfo
    static constexpr int QK = SI + NSTAGE * (int)sizeof(StageInfo);  // [QB][2*DK] f32
    static constexpr int PART = QK + QB * 2 * DK * 4;                // [NTEAMS][2][TEAM_WARPS] f32
    static constexpr int FLAG = PART + round_up(NTEAMS * 2 * TEAM_WARPS * 4, 16);
    static constexpr int RING = FLAG + 16;                           // [kRing] int: relayed group indices
    static constexpr int BARS = RING + kRing * 4;  // full, empty, conv, pub [NSTAGE]; qk [QB]; ring [kRing]
    static constexpr int TOTAL = BARS + (4 * NSTAGE + QB + kRing) * 8;
    static_assert(CG >= 1 && RG >= 1 && RPL >= 4 && (RPL & (RPL - 1)) == 0 && RG * CG == 32, "consumer geometry");
    static_assert(TOTAL <= 232448, "shared memory");
    static_assert(NSTAGE >= NTEAMS, "a team's previous unit of a stage is issued before its next one");
};

template <int DK, int DV>
__global__ void __launch_bounds__(WS<DK, DV>::NT, 1)
decode_ws_kernel(const DecodeArgs p, const int ncl) {
    using L = WS<DK, DV>;
    constexpr int NSTAGE = L::NSTAGE, QB = L::QB;
    extern __shared__ __align__(128) unsigned char smem[];
    float* tiles = reinterpret_cast<float*>(smem + L::TILES);
    uint16_t* zb = reinterpret_cast<uint16_t*>(smem + L::ZB);
    float* vsb = reinterpret_cast<float*>(smem + L::VS);
    StageInfo* si = reinterpret_cast<StageInfo*>(smem + L::SI);
    float* qkb = reinterpret_cast<float*>(smem + L::QK);
    float* part = reinterpret_cast<float*>(smem + L::PART);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::FLAG);
    // the last unit whose full barrier the first finisher warp has arrived on (for a CTA
    // that gives up: the arrivals that never came)
    volatile int* fin_full = abort_flag + 1;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
    uint64_t* empty = full + NSTAGE;
    uint64_t* cbar = empty + NSTAGE;
    uint64_t* pub = cbar + NSTAGE;
    uint64_t* qkbar = pub + NSTAGE;
    uint64_t* rbar = qkbar + QB;
    int* ring = reinterpret_cast<int*>(smem + L::RING);

    const int Hk = p.sh.Hk, Hv = p.sh.Hv, G = Hv / Hk, C = p.sh.C, W = p.sh.W;
    const int rank = (int)cluster_ctarank(), cid = blockIdx.x / G;
    const int ngroups_max = p.B * Hk;  // the launch's bound; the batch itself is read after the grid dependency
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(full + s, 2);  // the loader's copies (tile, z) and the finisher's "q/k are in" arrival
            mbar_init(pub + s, 1);   // the finisher's norms, k.q and gates
            mbar_init(empty + s, L::TEAM_WARPS);   // one arrival per warp of the consuming team
            mbar_init(cbar + s, 1);                // the staged conv inputs
        }
        for (int q = 0; q < QB; ++q) mbar_init(qkbar + q, 1);
        for (int r = 0; r < kRing; ++r) mbar_init(rbar + r, 1);
        *abort_flag = 0;
        *fin_full = -1;
        mbar_init_fence();
    }
    __syncthreads();
    int armed = 0;  // loader: units whose full and conv barriers it has armed
    auto fail = [&]() {
        if (lane == 0) {
            *abort_flag = 1;
            if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
        }
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait_deadline(bar, parity, kWaitTimeoutCycles, [&] { return *abort_flag != 0; });
    };
    auto slot_ok = [&](int s) { return s >= 0 && s < p.P; };

    // This CTA's conv channels, in local order: its share of the k-head's q/k
    // channels, then its v-head's v channels. They form at most three runs of
    // consecutive pool channels (q, k, v), each staged by bulk copies.
    const int qk_lo = (rank * 2 * DK) / G, nqk = (2 * DK) / G, nch = nqk + DV;
    const int nseg = G == 1 ? 3 : 2;
    auto seg_info = [&](int sg, int hk, int h, int& lc, int& ch, int& cnt) {
        if (G == 1 && sg < 2) {
            lc = sg * DK;
            ch = sg * Hk * DK + hk * DK;
            cnt = DK;
        } else if (sg == 0) {
            lc = 0;
            ch = qk_lo < DK ? hk * DK + qk_lo : Hk * DK + hk * DK + (qk_lo - DK);
            cnt = nqk;
        } else {
            lc = nqk;
            ch = 2 * Hk * DK + h * DV;
            cnt = DV;
        }
    };
    float* gparams = reinterpret_cast<float*>(smem + L::GP);  // A_log then dt_bias

    // With programmatic dependent launch this grid may start while the previous one
    // drains, so the state tiles of the fixed units are prefetched into L2 now (the
    // small conv inputs gain nothing from it). The slot read here may be stale (the
    // previous grid may still write the slot list): it only steers the hint, and L2
    // stays coherent with whatever that grid still writes. Nothing is read for use
    // before that grid has completed.
    if (warp == 0 && lane < 4 * kFixedUnits) {
        const int g = cid + (lane >> 2) * ncl;
        if (g < ngroups_max) {
            const int sl = __ldcg(p.slots + g / Hk);
            if (sl >= 0 && sl < p.P) {
                const char* t = reinterpret_cast<const char*>(
                    p.state_pool + ((size_t)sl * Hv + (g % Hk) * G + rank) * (size_t)(DK * DV));
                bulk_prefetch_l2(t + (lane & 3) * (L::TILE_BYTES / 4), L::TILE_BYTES / 4);
            }
        }
    }
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int ngroups = launch_batch(p.B_dev, p.B, p.err_flag, blockIdx.x == 0 && tid == 0) * Hk;
    // lane u of the loader: the slot of fixed unit u, loaded while the cluster barrier completes
    const int slot_fixed =
        warp == 0 && lane < kFixedUnits && cid + lane * ncl < ngroups ? __ldg(p.slots + (cid + lane * ncl) / Hk) : -1;
    cluster_arrive_relaxed();  // every CTA of the cluster runs before any st.async targets it
    cluster_wait_acquire();

    if (warp == 0) {
        // ============================== loader ==============================
        // Unit v's copies into stage v % NSTAGE as soon as the stage is free: the
        // state tile and z row (completing on full), the conv inputs and the a/b
        // groups (completing on cbar). The group and slot go along in the stage info.
        //
        // Which group unit v is: with a static schedule cid + v * ncl; with the
        // dynamic schedule the fixed units are the same, and after them the cluster's
        // rank 0 takes the group of unit v + 1 from the shared counter once unit v's
        // copies are out and relays it to every CTA of the cluster with st.async (ring
        // of kRing entries), so the CTAs of a cluster walk the same groups and faster
        // clusters simply take more of them.
        const int conv_bytes = 2 * W * nch * 2 + 32;
        const bool dyn = p.sched != nullptr;
        auto relay = [&](int v, unsigned int val) {  // rank 0, lane 0: the group of unit v >= kFixedUnits
            const int e = v - kFixedUnits;
            const uint32_t a_loc = smem_addr(ring + (e % kRing)), b_loc = smem_addr(rbar + (e % kRing));
            for (int r = 0; r < G; ++r)
                st_async_f32(cluster_map_u32(a_loc, r), __uint_as_float(val), cluster_map_u32(b_loc, r));
        };
        auto fetch = [&]() { return atomicAdd(p.sched, 1u); };
        auto receive = [&](int v) {  // lane-uniform group index of unit v (kEndOfWork past the end)
            int g;
            if (!dyn || v < kFixedUnits) {
                g = cid + v * ncl;
            } else {  // later units travel as ring entry v - kFixedUnits
                const int e = v - kFixedUnits;
                bool ok = true;
                if (lane == 0) {
                    mbar_arrive_expect_tx(rbar + (e % kRing), 4);
                    ok = wait(rbar + (e % kRing), (e / kRing) & 1);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) return -2;
                g = ring[e % kRing];
            }
            return g < ngroups ? g : kEndOfWork;
        };
        int g_next = receive(0);
        int slot_next = __shfl_sync(0xffffffffu, slot_fixed, 0);
        for (int v = 0;; ++v) {
            const int g = g_next, slot = slot_next;
            if (g == -2) {
                fail();
                break;
            }
            if (g == kEndOfWork) {  // one end marker per consumer team
                bool ok = true;
                for (int e = 0; e < L::NTEAMS && ok; ++e) {
                    const int ve = v + e, s = ve % NSTAGE;
                    if (ve >= NSTAGE && !wait(empty + s, ((ve / NSTAGE) - 1) & 1)) ok = false;
                    if (ok && lane == 0) {
                        si[s].group = kEndOfWork;
                        mbar_arrive(cbar + s);
                        mbar_arrive(full + s);
                        mbar_arrive(full + s);
                    }
                    __syncwarp();
                }
                if (!ok) fail();
                break;
            }
            const int s = v % NSTAGE, seq = g / Hk, hk = g - seq * Hk, h = hk * G + rank;
            if (v >= NSTAGE && !wait(empty + s, ((v / NSTAGE) - 1) & 1)) {
                fail();
                break;
            }
            const bool valid = slot_ok(slot);
            if (lane == 0) {
                si[s].group = g;
                si[s].slot = valid ? slot : -1;
                if (valid) {
                    mbar_arrive_expect_tx(full + s, L::TILE_BYTES + DV * 2);
                    mbar_arrive_expect_tx(cbar + s, conv_bytes);
                } else {
                    mbar_arrive(full + s);
                    mbar_arrive(cbar + s);
                }
            }
            armed = v + 1;
            __syncwarp();
            if (valid) {
                constexpr int nchunk = (L::TILE_BYTES + kTileChunk - 1) / kTileChunk;
                const char* src =
                    reinterpret_cast<const char*>(p.state_pool + ((size_t)slot * Hv + h) * (size_t)(DK * DV));
                char* dst = reinterpret_cast<char*>(tiles) + (size_t)s * L::TILE_BYTES;
                unsigned char* cst = smem + L::CONV + s * L::CSTAGE;
                // the small conv inputs first: the finishers need them long before the
                // consumers need the tile
                if (lane == 30 || lane == 31) {  // the 8-aligned group of a (lane 30) or b (lane 31) holding h
                    const uint16_t* srcab = (lane == 30 ? p.a : p.b) + (size_t)seq * Hv + (h & ~7);
                    tma_load_1d(smem + L::AB + s * 32 + (lane - 30) * 16, srcab, 16, cbar + s);
                } else if (lane < nseg * (W + 1)) {
                    const int sg = lane / (W + 1), kind = lane - sg * (W + 1);
                    int lc, ch, cnt;
                    seg_info(sg, hk, h, lc, ch, cnt);
                    if (kind < W - 1) {
                        tma_load_1d(cst + (kind * nch + lc) * 2,
                                    p.conv_pool + ((size_t)slot * (W - 1) + kind) * C + ch, cnt * 2, cbar + s);
                    } else if (kind == W - 1) {
                        tma_load_1d(cst + ((W - 1) * nch + lc) * 2, p.qkv + (size_t)seq * C + ch, cnt * 2, cbar + s);
                    } else {
                        tma_load_1d(cst + round_up(W * nch * 2, 16) + lc * W * 2, p.conv_w + (size_t)ch * W,
                                    cnt * W * 2, cbar + s);
                    }
                }
                __syncwarp();
                if (lane < nchunk) {
                    const int c = lane * kTileChunk;
                    tma_load_1d(dst + c, src + c, (uint32_t)min(kTileChunk, L::TILE_BYTES - c), full + s);
                } else if (lane == nchunk) {
                    tma_load_1d(zb + s * DV, p.z + ((size_t)seq * Hv + h) * DV, DV * 2, full + s);
                }
            }
            // The next unit's group and slot, while this unit's copies are in flight. With
            // the dynamic schedule the counter numbers the groups after the fixed ones; a
            // group is taken only once this unit's copies are out, so no cluster holds
            // more than the units its stages can take when the counter runs out.
            if (dyn && v + 1 >= kFixedUnits && rank == 0 && lane == 0)
                relay(v + 1, (unsigned)(kFixedUnits * ncl) + fetch());
            g_next = receive(v + 1);
            slot_next = v + 1 < kFixedUnits ? __shfl_sync(0xffffffffu, slot_fixed, v + 1)
                                            : (g_next >= 0 ? __ldg(p.slots + g_next / Hk) : -1);
        }
        // The last loader through leaves the counters at zero for the next call: every
        // fetch of every cluster has returned (its value was relayed) before its CTA
        // counts itself here, and nothing else in this launch reads the counters.
        if (dyn && lane == 0 && atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    } else if (warp <= L::FINISHER_WARPS) {
        // ============================== finishers ==============================
        // Units in order once their conv inputs have landed. All finisher warps
        // convolve this CTA's channels two at a time (step 3), send the raw q/k
        // share to every CTA of the cluster, keep v and roll the history; then the
        // first finisher warp waits for the other shares and publishes the norms, k.q
        // and the gates. A finisher warp runs at most one unit ahead of the first.
        const int fw = warp - 1;
        constexpr int NFT = 32 * L::FINISHER_WARPS;
        if (fw == 0) {
            for (int i = lane; i < Hv; i += 32) {
                gparams[i] = p.A_log[i];
                gparams[L::MAX_HV + i] = p.dt_bias[i];
            }
        }
        named_barrier(15, NFT);
        for (int v = 0;; ++v) {
            const int s = v % NSTAGE, q = v % QB;
            bool ok = wait(cbar + s, (v / NSTAGE) & 1);
            if (!ok) fail();
            if (!named_barrier_and(15, NFT, ok && !*abort_flag)) break;  // every finisher warp leaves together
            const int g = si[s].group;
            if (g == kEndOfWork) break;
            const int hk = g % Hk, h = hk * G + rank;
            const int slot = si[s].slot;
            const bool valid = slot >= 0;
            if (valid) {
                const unsigned char* cst = smem + L::CONV + s * L::CSTAGE;
                const uint16_t* rows = reinterpret_cast<const uint16_t*>(cst);
                const uint16_t* wts = reinterpret_cast<const uint16_t*>(cst + round_up(W * nch * 2, 16));
                uint16_t* hist = p.conv_pool + (size_t)slot * (W - 1) * C;
                const uint32_t q_loc = smem_addr(qkb + q * 2 * DK + qk_lo), bar_loc = smem_addr(qkbar + q);
                for (int c = 2 * (fw * 32 + lane); c < nch; c += 2 * NFT) {
                    // the two channels' weights are 2W consecutive bf16 values (W words):
                    // taps of channel c, then taps of channel c+1
                    float w0[kMaxConvWidthPersistent] = {0.f, 0.f, 0.f, 0.f};
                    float w1[kMaxConvWidthPersistent] = {0.f, 0.f, 0.f, 0.f};
                    auto lo = [](uint32_t x) { return bf16_bits_to_float(x & 0xffffu); };
                    auto hi = [](uint32_t x) { return bf16_bits_to_float(x >> 16); };
                    const uint32_t* wq = reinterpret_cast<const uint32_t*>(wts) + (c * W) / 2;
                    if (W == 4) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(wq);
                        w0[0] = lo(w4.x); w0[1] = hi(w4.x); w0[2] = lo(w4.y); w0[3] = hi(w4.y);
                        w1[0] = lo(w4.z); w1[1] = hi(w4.z); w1[2] = lo(w4.w); w1[3] = hi(w4.w);
                    } else if (W == 3) {
                        const uint32_t a0 = wq[0], a1 = wq[1], a2 = wq[2];
                        w0[0] = lo(a0); w0[1] = hi(a0); w0[2] = lo(a1);
                        w1[0] = hi(a1); w1[1] = lo(a2); w1[2] = hi(a2);
                    } else {
                        const uint32_t a0 = wq[0], a1 = wq[1];
                        w0[0] = lo(a0); w0[1] = hi(a0);
                        w1[0] = lo(a1); w1[1] = hi(a1);
                    }
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int j = 0; j < kMaxConvWidthPersistent; ++j) {
                        if (j < W) {
                            const uint32_t xx = *reinterpret_cast<const uint32_t*>(rows + j * nch + c);
                            acc0 = fmaf(w0[j], lo(xx), acc0);
                            acc1 = fmaf(w1[j], hi(xx), acc1);
                        }
                    }
                    const float s0 = silu(acc0), s1 = silu(acc1);
                    int lc, ch, cnt;
                    const int sg = G == 1 ? (c < DK ? 0 : (c < 2 * DK ? 1 : 2)) : (c < nqk ? 0 : 1);
                    seg_info(sg, hk, h, lc, ch, cnt);
                    ch += c - lc;
                    if (c < nqk) {
                        for (int r = 0; r < G; ++r)
                            st_async_f32x2(cluster_map_u32(q_loc + 4 * c, r), s0, s1, cluster_map_u32(bar_loc, r));
                    } else {
                        *reinterpret_cast<float2*>(vsb + s * DV + (c - nqk)) = make_float2(s0, s1);
                    }
                    for (int r = 0; r < W - 1; ++r)
                        *reinterpret_cast<uint32_t*>(hist + (size_t)r * C + ch) =
                            *reinterpret_cast<const uint32_t*>(rows + (r + 1) * nch + c);
                }
            }
            named_barrier(15, NFT);  // every finisher's v values are written
            if (fw != 0) continue;
            if (lane == 0) {
                if (valid) mbar_arrive_expect_tx(qkbar + q, 2 * DK * 4);
                else mbar_arrive(qkbar + q);
            }
            if (!wait(qkbar + q, (v / QB) & 1)) {
                fail();  // the other finisher warps see the abort at the next agreement
                continue;
            }
            if (lane == 0) {
                mbar_arrive(full + s);  // the raw q/k and v are in: pass 1 may start
                *fin_full = v;
            }
            if (valid) {
                const float* qr = qkb + q * 2 * DK;
                float sq = 0.f, sk = 0.f, dot = 0.f;
                for (int i = lane; i < DK; i += 32) {
                    const float a = qr[i], b = qr[DK + i];
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
                    StageInfo& st = si[s];
                    st.nq = rsqrtf(sq + p.sh.l2_eps) * p.sh.q_scale;
                    st.nk = rsqrtf(sk + p.sh.l2_eps);
                    st.kq = dot * st.nq * st.nk;
                    const uint16_t* ab = reinterpret_cast<const uint16_t*>(smem + L::AB + s * 32);
                    gate_and_beta(ab[h & 7], ab[8 + (h & 7)], gparams[h], gparams[L::MAX_HV + h], st.alpha,
                                  st.beta);
                }
            } else if (lane == 0 && p.err_flag) {
                atomicOr(p.err_flag, GDN_DEVICE_ERR_SLOT_RANGE_BIT);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(pub + s);
        }
    } else {
        // ============================== consumers ==============================
        const int cw = warp - L::PRODUCER_WARPS, team = cw / L::TEAM_WARPS, wt = cw - team * L::TEAM_WARPS;
        const int rg = lane / L::CG, cg = lane - rg * L::CG;
        const int col = wt * L::CPW + 4 * cg;
        int parity_part = 0;
        for (int u = team;; u += L::NTEAMS) {
            const int s = u % NSTAGE, q = u % QB;
            // The teams take units in turn, so the stage's previous unit may be another team's
            // and still incomplete (its tile landing); a parity wait on the full barrier two
            // phases ahead would then pass at once. The previous unit's release comes first: it
            // is at most one phase away (the loader has issued that unit, this team having
            // passed a later one), and the loader waited on the same phase before issuing this
            // unit's copies, so it costs nothing once the full barrier can complete.
            bool ok = u < NSTAGE || wait(empty + s, ((u / NSTAGE) - 1) & 1);
            ok = ok && wait(full + s, (u / NSTAGE) & 1);
            if (!ok) fail();
            if (L::TEAM_WARPS > 1) ok = named_barrier_and(1 + team, 32 * L::TEAM_WARPS, ok && !*abort_flag);
            else ok = __all_sync(0xffffffffu, ok && !*abort_flag);
            if (!ok) break;  // the team's warps leave together
            const int st_group = si[s].group, st_slot = si[s].slot;
            if (st_group == kEndOfWork) break;
            if (st_slot >= 0) {
                const int seq = st_group / Hk, h = (st_group - seq * Hk) * G + rank;
                const uint2 zz = rg == 0 ? *reinterpret_cast<const uint2*>(zb + s * DV + col) : make_uint2(0u, 0u);
                const float4* tl = reinterpret_cast<const float4*>(tiles + (size_t)s * (DK * DV)) + col / 4;
                const float* qr = qkb + q * 2 * DK;
                const float* kr = qr + DK;
                const int row0 = rg * L::RPL;  // this lane's rows: row0 .. row0 + RPL - 1
                float4 mk = make_float4(0.f, 0.f, 0.f, 0.f), mq = mk;
                // each row group starts its rows at a different offset, so the four
                // groups read k and q from different banks
                const int rot = 4 * rg;
#pragma unroll 2
                for (int i = 0; i < L::RPL; i += 4) {
                    const int r = row0 + ((i + rot) & (L::RPL - 1));
                    const float4 k4 = *reinterpret_cast<const float4*>(kr + r);
                    const float4 q4 = *reinterpret_cast<const float4*>(qr + r);
                    const float kk[4] = {k4.x, k4.y, k4.z, k4.w}, qq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 x = tl[(size_t)(r + e) * (DV / 4)];
                        mk.x = fmaf(x.x, kk[e], mk.x); mk.y = fmaf(x.y, kk[e], mk.y);
                        mk.z = fmaf(x.z, kk[e], mk.z); mk.w = fmaf(x.w, kk[e], mk.w);
                        mq.x = fmaf(x.x, qq[e], mq.x); mq.y = fmaf(x.y, qq[e], mq.y);
                        mq.z = fmaf(x.z, qq[e], mq.z); mq.w = fmaf(x.w, qq[e], mq.w);
                    }
                }
#pragma unroll
                for (int off = L::CG; off < 32; off <<= 1) {
                    mk.x += __shfl_xor_sync(0xffffffffu, mk.x, off); mk.y += __shfl_xor_sync(0xffffffffu, mk.y, off);
                    mk.z += __shfl_xor_sync(0xffffffffu, mk.z, off); mk.w += __shfl_xor_sync(0xffffffffu, mk.w, off);
                    mq.x += __shfl_xor_sync(0xffffffffu, mq.x, off); mq.y += __shfl_xor_sync(0xffffffffu, mq.y, off);
                    mq.z += __shfl_xor_sync(0xffffffffu, mq.z, off); mq.w += __shfl_xor_sync(0xffffffffu, mq.w, off);
                }
                const float4 vv = *reinterpret_cast<const float4*>(vsb + s * DV + col);
                // the norms, k.q and gates of this unit (published after the q/k exchange)
                bool okp = wait(pub + s, (u / NSTAGE) & 1);
                if (!okp) fail();
                if (L::TEAM_WARPS > 1) okp = named_barrier_and(1 + team, 32 * L::TEAM_WARPS, okp && !*abort_flag);
                else okp = __all_sync(0xffffffffu, okp && !*abort_flag);
                if (!okp) break;
                const StageInfo st = si[s];
                const float am = st.alpha * st.nk, aq = st.alpha * st.nq;
                float4 d, o;
                d.x = st.beta * fmaf(-am, mk.x, vv.x); d.y = st.beta * fmaf(-am, mk.y, vv.y);
                d.z = st.beta * fmaf(-am, mk.z, vv.z); d.w = st.beta * fmaf(-am, mk.w, vv.w);
                o.x = fmaf(aq, mq.x, d.x * st.kq); o.y = fmaf(aq, mq.y, d.y * st.kq);
                o.z = fmaf(aq, mq.z, d.z * st.kq); o.w = fmaf(aq, mq.w, d.w * st.kq);
                const float4 dn = make_float4(d.x * st.nk, d.y * st.nk, d.z * st.nk, d.w * st.nk);
                // the updated rows go straight to the pool (streaming stores: nothing here reads them again)
                float4* sg = reinterpret_cast<float4*>(p.state_pool + ((size_t)st_slot * Hv + h) * (size_t)(DK * DV)) +
                             col / 4;
#pragma unroll 2
                for (int i = 0; i < L::RPL; i += 4) {
                    const int r = row0 + ((i + rot) & (L::RPL - 1));
                    const float4 k4 = *reinterpret_cast<const float4*>(kr + r);
                    const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float4 x = tl[(size_t)(r + e) * (DV / 4)];
                        x.x = fmaf(st.alpha, x.x, kk[e] * dn.x); x.y = fmaf(st.alpha, x.y, kk[e] * dn.y);
                        x.z = fmaf(st.alpha, x.z, kk[e] * dn.z); x.w = fmaf(st.alpha, x.w, kk[e] * dn.w);
                        __stcs(sg + (size_t)(r + e) * (DV / 4), x);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + s);
                // ---- step 8 over the whole head: the team's warps pool their sums of o^2
                float ss = rg == 0 ? o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w : 0.f;
#pragma unroll
                for (int off = 1; off < L::CG; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                float* pt = part + (team * 2 + parity_part) * L::TEAM_WARPS;
                if (lane == 0) pt[wt] = ss;
                if (L::TEAM_WARPS > 1) named_barrier(1 + team, 32 * L::TEAM_WARPS);
                else __syncwarp();
                float tot = 0.f;
#pragma unroll
                for (int w = 0; w < L::TEAM_WARPS; ++w) tot += pt[w];
                if (rg == 0) {
                    const float inv = rsqrtf(tot / (float)DV + p.sh.rms_eps);
                    const uint2 ww = *reinterpret_cast<const uint2*>(p.norm_w + col);
                    const float y0 = o.x * inv * bf16_bits_to_float(ww.x & 0xffffu) * silu(bf16_bits_to_float(zz.x & 0xffffu));
                    const float y1 = o.y * inv * bf16_bits_to_float(ww.x >> 16) * silu(bf16_bits_to_float(zz.x >> 16));
                    const float y2 = o.z * inv * bf16_bits_to_float(ww.y & 0xffffu) * silu(bf16_bits_to_float(zz.y & 0xffffu));
                    const float y3 = o.w * inv * bf16_bits_to_float(ww.y >> 16) * silu(bf16_bits_to_float(zz.y >> 16));
                    const size_t oi = ((size_t)seq * Hv + h) * DV + col;
                    uint2 packed;
                    packed.x = (uint32_t)float_to_bf16_bits(y0) | ((uint32_t)float_to_bf16_bits(y1) << 16);
                    packed.y = (uint32_t)float_to_bf16_bits(y2) | ((uint32_t)float_to_bf16_bits(y3) << 16);
                    *reinterpret_cast<uint2*>(p.out + oi) = packed;
                    if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + oi) = make_float4(y0, y1, y2, y3);
                }
                parity_part ^= 1;
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + s);
            }
        }
    }
    __syncthreads();
    // A wait gave up: before the CTA leaves, the copies it still has in flight land (or a
    // further bounded wait runs out). Every role has left its loop, so nothing else arrives
    // on these barriers now. A stage is re-armed only after its previous phase completed,
    // so only the last NSTAGE armed units can be outstanding; the conv barrier counts the
    // loader's arrival and its copies, the full barrier also the first finisher warp's
    // arrival, which is made here where it never came.
    if (warp == 0 && lane == 0 && *abort_flag) {
        for (int v = armed > NSTAGE ? armed - NSTAGE : 0; v < armed; ++v) {
            const int s = v % NSTAGE;
            const uint32_t par = (uint32_t)((v / NSTAGE) & 1);
            mbar_wait_bounded(cbar + s, par);
            if (v > *fin_full) mbar_arrive(full + s);
            mbar_wait_bounded(full + s, par);
        }
    }
    // No CTA leaves while a peer may still send to it. Every message a CTA expects has
    // been waited for, so the arrival needs no release ordering of this CTA's stores.
    cluster_arrive_relaxed();
    cluster_wait_acquire();
}

template <int DK, int DV>
cudaError_t launch_ws_tile(const DecodeArgs& a, int G, cudaStream_t stream, bool query_only, int* cap_out) {
    using L = WS<DK, DV>;
    auto kern = decode_ws_kernel<DK, DV>;
    // co-resident clusters per (device, cluster size), queried once; threads may race to
    // fill an entry, and all of them store the same value
    static std::atomic<int> cap_cache[kMaxDevices][9];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(L::NT);
    cfg.dynamicSmemBytes = L::TOTAL;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;  // the occupancy query takes the cluster shape only
    int cap = cap_cache[dev][G].load(std::memory_order_relaxed);
    if (cap <= 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3((unsigned)G);
        int maxc = 0;
        e = cudaOccupancyMaxActiveClusters(&maxc, kern, &cfg);
        if (e != cudaSuccess) return e;
        cap = maxc;
        cap_cache[dev][G].store(maxc, std::memory_order_relaxed);
    }
    if (cap_out) *cap_out = cap;
    if (query_only) return cudaSuccess;
    const int ngroups = a.B * a.sh.Hk;
    const int ncl = ngroups < cap ? ngroups : cap;  // the dynamic schedule needs ncl <= co-resident clusters too
    if (ncl <= 0) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)(ncl * G));
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a, ncl);
}

template <int DK>
cudaError_t ws_dispatch(const DecodeArgs& a, int G, cudaStream_t stream, bool query_only, int* cap) {
    switch (a.sh.dv) {
        case 16:
            if constexpr (DK >= 32) return launch_ws_tile<DK, 16>(a, G, stream, query_only, cap);
            return cudaErrorInvalidValue;
        case 32: return launch_ws_tile<DK, 32>(a, G, stream, query_only, cap);
        case 64: return launch_ws_tile<DK, 64>(a, G, stream, query_only, cap);
        case 128: return launch_ws_tile<DK, 128>(a, G, stream, query_only, cap);
    }
    return cudaErrorInvalidValue;
}

cudaError_t ws_call(const DecodeArgs& a, cudaStream_t stream, bool query_only, int* cap) {
    const int G = a.sh.Hv / a.sh.Hk;
    if (!persistent_supported(a)) return cudaErrorInvalidValue;
    switch (a.sh.dk) {
        case 16: return ws_dispatch<16>(a, G, stream, query_only, cap);
        case 32: return ws_dispatch<32>(a, G, stream, query_only, cap);
        case 64: return ws_dispatch<64>(a, G, stream, query_only, cap);
        case 128: return ws_dispatch<128>(a, G, stream, query_only, cap);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool persistent_supported(const DecodeArgs& a) {
    // the q/k share of each CTA must be a whole number of 16-byte bf16 runs for the
    // bulk copies of the conv inputs
    const int G = a.sh.Hv / a.sh.Hk;
    return a.T == 1 && a.sh.W <= kMaxConvWidthPersistent && G <= 8 && (2 * a.sh.dk) % (8 * G) == 0 &&
           a.sh.Hv % 8 == 0 && a.sh.Hv <= 128 && (a.sh.dv >= 32 || a.sh.dk >= 32);
}

cudaError_t persistent_capacity(const DecodeArgs& a, int* max_clusters) {
    return ws_call(a, nullptr, true, max_clusters);
}

cudaError_t launch_decode_persistent(const DecodeArgs& a, cudaStream_t stream) {
    return ws_call(a, stream, false, nullptr);
}

}  // namespace gdn
