// The projections on either side of the GDN decode step, on the fifth-generation
// tensor cores: step 2 of the page "spark_model/forward/qwen3_5/linear_attention.rs"
// (in_proj_qkv, in_proj_z and the dual-output in_proj_a / in_proj_b GEMVs, all
// reading the same normalised input x_norm, here ONE GEMM over the four weights
// stacked row-wise) and the GEMV of its fused steps 9+10+11 (out_proj applied to the
// SiLU(z)-gated, normalised output, which the decode step already produces).
//
// D[r][n] = sum_k X[r][k] W[n][k] for token rows r < R <= 256 and output features n:
// a skinny GEMM whose cost is the weight bytes. It runs with the operands swapped,
// D^T = W X^T, so the MMA's M = 128 rows are weight rows (output features) and its N
// is the token rows padded to a multiple of 16: no MMA lane is wasted on padding at
// decode batch sizes.
//
// Grid: ceil(N/128) weight tiles x S K-slices; the S CTAs of a tile form a thread-block
// cluster (S <= 8). A CTA of 128 threads:
//  * thread 0 issues the TMA tile loads (128 B swizzle, no multicast) of its K-slice
//    into a ring of NSTAGE stages, each a 128 x 64 weight tile and an Rp x 64 X tile;
//  * thread 32 issues tcgen05.mma (kind::f16, bf16 in, fp32 accumulate in TMEM), four
//    K=16 steps per stage, and frees each stage with tcgen05.commit;
//  * after the last MMA all four warps read the accumulator (warp w owns TMEM lanes
//    32w..32w+31, i.e. weight rows) into shared memory; the cluster then sums its S
//    partial tiles over distributed shared memory in rank order (deterministic), CTA
//    rank q taking a band of rows, and stores bf16 (and optionally fp32) outputs.
// Every mbarrier wait is bounded by the SM cycle counter; on expiry the CTA records
// GDN_DEVICE_ERR_TIMEOUT, stops issuing work, lets what it issued complete, frees
// its TMEM and leaves through the cluster barriers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "gdn_device.cuh"
#include "gdn_internal.h"
#include "gdn_tcgen05.cuh"

namespace gdn {
namespace {

constexpr int kTileN = 128;      // weight rows per tile (the MMA's M)
constexpr int kTileK = 64;       // bf16 elements per 128-byte swizzled row
#ifndef GDN_PROJ_STAGES
#define GDN_PROJ_STAGES 4
#endif
constexpr int kStages = GDN_PROJ_STAGES;  // stages in flight per CTA (build-time tuning)
// 64-element K sub-tiles per stage: a stage reads kSub * 128 contiguous bytes of every
// weight row it covers (build-time tuning)
#ifndef GDN_PROJ_SUB
#define GDN_PROJ_SUB 1
#endif
constexpr int kSub = GDN_PROJ_SUB;
constexpr int kBlockK = kSub * 64;  // K elements per stage
constexpr int kThreads = 128;
constexpr int kMaxSlices = 8;    // portable cluster size
constexpr int kWBytes = kTileN * kTileK * 2;  // 16 KiB

__host__ __device__ constexpr int rows_padded(int R) { return (R + 15) / 16 * 16; }
__host__ __device__ constexpr int sub_bytes(int Rp) { return kWBytes + Rp * kTileK * 2; }  // one K sub-tile
__host__ __device__ constexpr int stage_bytes(int Rp) { return kSub * sub_bytes(Rp); }
// the partial tile of the cluster reduction: [128][Rp + 4] fp32 (padded rows)
__host__ __device__ constexpr int red_stride(int Rp) { return Rp + 4; }
__host__ __device__ constexpr int smem_bytes(int Rp) {
    const int ring = kStages * stage_bytes(Rp);
    const int red = kTileN * red_stride(Rp) * 4;
    return 1024 + (ring > red ? ring : red) + 128;  // alignment slack, ring (reused), barriers
}

// ---- PTX wrappers (tcgen05, TMA tiles)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];\n"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTileN >> 4) << 24);
}

__global__ void __launch_bounds__(kThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                 const ProjArgs p) {
    extern __shared__ unsigned char smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.slices, rank = (int)cluster_ctarank();
    const int tile = blockIdx.x / S;
    const int Rp = rows_padded(p.R);
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - smem_addr(smem_raw));
    const int sbytes = stage_bytes(Rp);
    const int ring = kStages * sbytes, red = kTileN * red_stride(Rp) * 4;
    unsigned char* ctl = gbase + (ring > red ? ring : red);
    uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t ncols = Rp <= 32 ? 32 : (Rp <= 64 ? 64 : (Rp <= 128 ? 128 : 256));

    // this CTA's K-slice, in 64-element blocks
    const int nkb = (p.K + kBlockK - 1) / kBlockK;
    const int kb0 = (int)((long)rank * nkb / S), kb1 = (int)((long)(rank + 1) * nkb / S);
    const int nk = kb1 - kb0;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    }
    if (warp == 1) tmem_alloc(smem_addr(tmem_slot), ncols);
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the inputs may be written by the kernel before this one in the stream
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    auto fail = [&]() {
        *abort_flag = 1;
        if (p.err_flag) atomicOr(p.err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait_deadline(bar, parity, kWaitTimeoutCycles, [&] { return *abort_flag != 0; });
    };

    int issued = 0;  // stages the loader armed (thread 0)
    if (tid == 0) {
        // ---- loader: weight tile rows tile*128.., token rows 0..Rp-1, K block kb
        for (int i = 0; i < nk; ++i) {
            const int s = i % kStages;
            if (i >= kStages && !wait(empty + s, ((i / kStages) - 1) & 1)) {
                fail();
                break;
            }
            const uint32_t st = base + s * sbytes;
            mbar_arrive_expect_tx(full + s, (uint32_t)sbytes);
            for (int j = 0; j < kSub; ++j) {  // sub-tile j: the next 64 K elements of the same rows
                const int kx = (kb0 + i) * kBlockK + j * kTileK;
                const uint32_t sj = st + j * sub_bytes(Rp);
                tma_load_2d(sj, &map_w, kx, tile * kTileN, smem_addr(full + s));
                tma_load_2d(sj + kWBytes, &map_x, kx, 0, smem_addr(full + s));
            }
            issued = i + 1;
        }
    } else if (tid == 32) {
        // ---- MMA issuer
        const uint32_t idesc = idesc_bf16(Rp);
        int i = 0;
        for (; i < nk; ++i) {
            const int s = i % kStages;
            if (!wait(full + s, (i / kStages) & 1)) {
                fail();
                break;
            }
            tcgen05_fence_after();
            const uint32_t st = base + s * sbytes;
            for (int j = 0; j < kSub; ++j) {
                const uint32_t sj = st + j * sub_bytes(Rp);
                const uint64_t da = sw128_desc(sj), db = sw128_desc(sj + kWBytes);
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk)  // K = 16 per MMA: 32 bytes along the swizzled row
                    umma_bf16(tmem, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk), idesc,
                              (i > 0 || j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(smem_addr(empty + s));  // the stage is free once these MMAs have read it
        }
        umma_commit(smem_addr(done));  // every MMA issued above has completed
    }
    // ---- accumulator -> shared memory (this CTA's partial tile), fp32 [128][Rp + 4]
    // Waited for on time only: whatever was issued completes (its operands are in), and
    // the TMEM it writes is freed only after that. CTA-uniform: the reads below are
    // warp-collective.
    const bool got = mbar_wait_bounded(done, 0);
    if (!got) fail();
    const bool ok_done = __syncthreads_and(got && !*abort_flag) != 0;
    tcgen05_fence_after();
    float* redp = reinterpret_cast<float*>(gbase);
    const int rs = red_stride(Rp);
    if (ok_done && nk > 0) {
        const int row = warp * 32 + lane;
        for (int c = 0; c < Rp; c += 16) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(redp + row * rs + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    } else {
        for (int i = tid; i < kTileN * rs; i += kThreads) redp[i] = 0.f;
    }
    // On an abort the loader's copies that nothing consumed must land before the
    // CTA's shared memory is reused or released.
    if (tid == 0 && *abort_flag) {
        for (int i = 0; i < issued; ++i) {
            const int s = i % kStages;
            if (i >= issued - kStages) wait(full + s, (i / kStages) & 1);
        }
    }
    tcgen05_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, ncols);
    cluster_arrive_release();  // every CTA's partial tile is in its shared memory
    cluster_wait_acquire();

    // ---- the cluster's sum, rank order; rank q stores rows [q*128/S, (q+1)*128/S)
    const int r0 = rank * kTileN / S, r1 = (rank + 1) * kTileN / S;
    const int nq = Rp / 4;  // float4 groups of token rows
    const uint32_t red_local = smem_addr(redp);
    for (int t = tid; t < (r1 - r0) * nq; t += kThreads) {
        const int g = t / (r1 - r0), row = r0 + (t - g * (r1 - r0));
        const int n = tile * kTileN + row;
        const int c = 4 * g;
        if (n >= p.N || c >= p.R) continue;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 0; q < S; ++q) {
            const float4 v = ld_cluster_f4(cluster_map_u32(red_local + (uint32_t)(row * rs + c) * 4u, q));
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        int width = p.seg_width[0], start = p.seg_start[0];
        uint16_t* dst = p.seg_out[0];
#pragma unroll
        for (int i = 1; i < 4; ++i)
            if (i < p.nseg && n >= p.seg_start[i]) {
                width = p.seg_width[i];
                start = p.seg_start[i];
                dst = p.seg_out[i];
            }
        const int col = n - start;
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = c + i;
            if (r < p.R) {
                dst[(size_t)r * width + col] = float_to_bf16_bits(vals[i]);
                if (p.out_f32) p.out_f32[(size_t)r * p.N + n] = vals[i];
            }
        }
    }
    cluster_arrive_release();  // no CTA leaves while a peer may still read its partial tile
    cluster_wait_acquire();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A 2D bf16 tensor map over rows x cols (row-major, cols contiguous) with boxes of
// box_rows x 64 and the 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The kernel's dynamic shared-memory limit, raised once per device to what the largest
// launch (256 token rows) needs.
cudaError_t proj_kernel_attribute() {
    static std::mutex mu;
    static bool set[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!set[dev]) {
        int optin = 0;
        if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return e;
        const int want = smem_bytes(rows_padded(kProjMaxRows));
        if ((e = cudaFuncSetAttribute(proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      want < optin ? want : optin)) != cudaSuccess)
            return e;
        set[dev] = true;
    }
    return cudaSuccess;
}

// Co-resident clusters of `s` CTAs for a launch of R token rows, queried once per
// (device, s, padded rows) and cached.
cudaError_t proj_cluster_capacity(int s, int R, int* out) {
    static std::mutex mu;
    struct Entry { int dev, s, rp, cap; };
    static Entry cache[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int rp = rows_padded(R);
    if ((e = proj_kernel_attribute()) != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (cache[i].dev == dev && cache[i].s == s && cache[i].rp == rp) {
            *out = cache[i].cap;
            return cudaSuccess;
        }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)s);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem_bytes(rp);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)s;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int cap = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&cap, proj_gemm_kernel, &cfg)) != cudaSuccess) return e;
    if (n < 256) cache[n++] = {dev, s, rp, cap};
    *out = cap;
    return cudaSuccess;
}

// K-slices per weight tile. With at least half as many weight tiles as SMs (in_proj's
// 97 at the benchmark shape) two slices measured fastest (17.7 against 20.6 µs unsplit;
// three and more did not fit one wave of clusters). With fewer tiles, the most slices (up
// to 8, at least two K blocks each) for which every tile's cluster is co-resident, so
// the launch is one wave (out_proj's 16 tiles: 6).
cudaError_t proj_slices(int N, int K, int R, int* slices) {
    const int tiles = (N + kTileN - 1) / kTileN, nkb = (K + kBlockK - 1) / kBlockK;
#ifdef GDN_PROJ_SLICES_OVERRIDE
    {  // build-time tuning override, used when the shape allows it
        const int s = GDN_PROJ_SLICES_OVERRIDE;
        if (s >= 1 && s <= kMaxSlices && s <= nkb) {
            *slices = s;
            return cudaSuccess;
        }
    }
#endif
    int dev = 0, sms = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e0 != cudaSuccess) return e0;
    if (2 * tiles >= sms && nkb >= 4) {
        *slices = 2;
        return cudaSuccess;
    }
    int best = 1;
    for (int s = 2; s <= kMaxSlices && 2 * s <= nkb; ++s) {
        int cap = 0;
        cudaError_t e = proj_cluster_capacity(s, R, &cap);
        if (e != cudaSuccess) return e;
        if (cap >= tiles) best = s;
    }
    *slices = best;
    return cudaSuccess;
}

int proj_smem_bytes(int R) { return smem_bytes(rows_padded(R)); }

cudaError_t launch_proj_gemm(const ProjArgs& a, cudaStream_t stream) {
    if (a.R <= 0 || a.N <= 0) return cudaSuccess;
    CUtensorMap mw, mx;
    if (!make_map(&mw, a.w, a.N, a.K, kTileN) || !make_map(&mx, a.x, a.R, a.K, rows_padded(a.R)))
        return cudaErrorInvalidValue;
    const int smem = smem_bytes(rows_padded(a.R));
    cudaError_t e = proj_kernel_attribute();
    if (e != cudaSuccess) return e;
    const int tiles = (a.N + kTileN - 1) / kTileN;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * a.slices));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)a.slices;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, proj_gemm_kernel, mw, mx, a);
}

}  // namespace gdn
