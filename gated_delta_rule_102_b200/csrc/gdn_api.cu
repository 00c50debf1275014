// C-ABI entry points of libgdn (declared in include/gdn.h). Every argument is checked
// here, on the host, before anything is enqueued, so an error return means nothing
// was written; then one launch per entry point goes onto the caller's stream.
// Following the "fail before the first launch" convention of the Metrale layer page
// ("metrale_model_arch/glm5next_dsa/layer.rs", its invariants paragraph).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "gdn.h"
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace {

bool supported_head_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

gdn_status check_config(const gdn_config* cfg, gdn::Shape* sh) {
    if (!cfg) return GDN_ERR_INVALID_ARGUMENT;
    if (cfg->num_k_heads <= 0 || cfg->num_v_heads <= 0 || cfg->head_k_dim <= 0 || cfg->head_v_dim <= 0 ||
        cfg->conv_width <= 0)
        return GDN_ERR_INVALID_ARGUMENT;
    if (cfg->num_v_heads % cfg->num_k_heads != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (!(cfg->l2_eps >= 0.0f) || !(cfg->rms_eps >= 0.0f) || !isfinite(cfg->l2_eps) || !isfinite(cfg->rms_eps) ||
        !isfinite(cfg->q_scale))
        return GDN_ERR_INVALID_ARGUMENT;
    if (cfg->num_v_heads / cfg->num_k_heads > 8) return GDN_ERR_UNSUPPORTED;
    if (!supported_head_dim(cfg->head_k_dim) || !supported_head_dim(cfg->head_v_dim)) return GDN_ERR_UNSUPPORTED;
    if (cfg->conv_width < 2 || cfg->conv_width > gdn::kMaxConvWidth) return GDN_ERR_UNSUPPORTED;
    const long C = 2L * cfg->num_k_heads * cfg->head_k_dim + (long)cfg->num_v_heads * cfg->head_v_dim;
    if (C > (1L << 30)) return GDN_ERR_UNSUPPORTED;
    sh->Hk = cfg->num_k_heads;
    sh->Hv = cfg->num_v_heads;
    sh->dk = cfg->head_k_dim;
    sh->dv = cfg->head_v_dim;
    sh->W = cfg->conv_width;
    sh->C = (int)C;
    sh->l2_eps = cfg->l2_eps;
    sh->rms_eps = cfg->rms_eps;
    sh->q_scale = cfg->q_scale != 0.0f ? cfg->q_scale : 1.0f / sqrtf((float)cfg->head_k_dim);
    return GDN_OK;
}

gdn_status check_batch(int32_t B, int32_t T, int32_t pool_slots, const gdn::Shape& sh) {
    if (B < 0 || T <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (T > gdn::kMaxTokens) return GDN_ERR_UNSUPPORTED;
    if (B > 0 && pool_slots <= 0) return GDN_ERR_INVALID_ARGUMENT;
    // grid: B * Hv * (at most 8 slices) CTAs
    if ((long)B * sh.Hv * 8 > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

// All pointers non-null and 16-byte aligned (nullable ones checked only when set).
gdn_status check_pointers(std::initializer_list<const void*> required, std::initializer_list<const void*> nullable) {
    for (const void* p : required)
        if (!p) return GDN_ERR_INVALID_ARGUMENT;
    for (const void* p : required)
        if (!aligned16(p)) return GDN_ERR_MISALIGNED;
    for (const void* p : nullable)
        if (p && !aligned16(p)) return GDN_ERR_MISALIGNED;
    return GDN_OK;
}

// Every check of gdn_decode_step, and its kernel arguments: nothing is enqueued here.
// B == 0 returns GDN_OK with `d` unset (the call is a no-op).
gdn_status check_decode(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv, const uint16_t* a,
                        const uint16_t* b, const uint16_t* z, const uint16_t* conv_w, const float* A_log,
                        const float* dt_bias, const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                        int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16, float* out_f32,
                        int32_t* err_flag, void* workspace, gdn::DecodeArgs* d) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_batch(B, T, pool_slots, sh)) != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((st = check_pointers({qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool, slots, out_bf16},
                             {out_f32, err_flag, workspace})) != GDN_OK)
        return st;
    const int G = sh.Hv / sh.Hk;
    *d = gdn::DecodeArgs{sh, B, T, pool_slots, gdn::decode_column_splits(B, sh.Hv, G, sh.dv),
                         qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool, slots,
                         out_bf16, out_f32, err_flag, static_cast<unsigned int*>(workspace)};
    return GDN_OK;
}

gdn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

// hidden: a multiple of 8 (16-byte rows for the tile copies); rows: 0..256 token rows.
gdn_status check_proj_sizes(int32_t hidden, int32_t rows) {
    if (hidden <= 0 || rows < 0) return GDN_ERR_INVALID_ARGUMENT;
    if (hidden % 8 != 0 || hidden > (1 << 20) || rows > gdn::kProjMaxRows) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status launch_proj(gdn::ProjArgs& p, cudaStream_t stream) {
    if (gdn::proj_slices(p.N, p.K, p.R, &p.slices) != cudaSuccess) return GDN_ERR_CUDA;
    return from_cuda(gdn::launch_proj_gemm(p, stream));
}

}  // namespace

extern "C" {

gdn_status gdn_conv_update(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv, const uint16_t* conv_w,
                           uint16_t* conv_pool, int32_t pool_slots, const int32_t* slots, float* q_out, float* k_out,
                           float* v_out, int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_batch(B, T, pool_slots, sh)) != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((st = check_pointers({qkv, conv_w, conv_pool, slots, q_out, k_out, v_out}, {err_flag})) != GDN_OK) return st;
    gdn::ConvArgs a{sh, B, T, pool_slots, qkv, conv_w, conv_pool, slots, q_out, k_out, v_out, err_flag};
    return from_cuda(gdn::launch_conv_update(a, (cudaStream_t)stream));
}

gdn_status gdn_recurrent_step(const gdn_config* cfg, int32_t B, int32_t T, const float* q, const float* k,
                              const float* v, const uint16_t* a, const uint16_t* b, const float* A_log,
                              const float* dt_bias, float* state_pool, int32_t pool_slots, const int32_t* slots,
                              float* o, int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_batch(B, T, pool_slots, sh)) != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((st = check_pointers({q, k, v, a, b, A_log, dt_bias, state_pool, slots, o}, {err_flag})) != GDN_OK)
        return st;
    gdn::RecurrentArgs r{sh, B, T, pool_slots, gdn::recurrent_column_splits(B, sh.Hv, sh.dv),
                         q, k, v, a, b, A_log, dt_bias, state_pool, slots, o, err_flag};
    return from_cuda(gdn::launch_recurrent(r, (cudaStream_t)stream));
}

gdn_status gdn_gated_rmsnorm(const gdn_config* cfg, int32_t rows, const float* o, const uint16_t* z,
                             const uint16_t* norm_w, uint16_t* out_bf16, float* out_f32, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if (rows < 0) return GDN_ERR_INVALID_ARGUMENT;
    if (rows == 0) return GDN_OK;
    if ((st = check_pointers({o, z, norm_w, out_bf16}, {out_f32})) != GDN_OK) return st;
    gdn::NormArgs n{sh, rows, o, z, norm_w, out_bf16, out_f32};
    return from_cuda(gdn::launch_gated_rmsnorm(n, (cudaStream_t)stream));
}

gdn_status gdn_decode_step(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv, const uint16_t* a,
                           const uint16_t* b, const uint16_t* z, const uint16_t* conv_w, const float* A_log,
                           const float* dt_bias, const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                           int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16, float* out_f32,
                           int32_t* err_flag, void* workspace, void* stream) {
    gdn::DecodeArgs d;
    gdn_status st = check_decode(cfg, B, T, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool,
                                 pool_slots, slots, out_bf16, out_f32, err_flag, workspace, &d);
    if (st != GDN_OK || B == 0) return st;
    return from_cuda(gdn::launch_decode_fused(d, (cudaStream_t)stream));
}

size_t gdn_decode_workspace_bytes(void) { return 64; }

gdn_status gdn_decode_step_device_batch(const gdn_config* cfg, const int32_t* B_dev, int32_t B_max, int32_t T,
                                        const uint16_t* qkv, const uint16_t* a, const uint16_t* b, const uint16_t* z,
                                        const uint16_t* conv_w, const float* A_log, const float* dt_bias,
                                        const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                                        int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16, float* out_f32,
                                        int32_t* err_flag, void* workspace, void* stream) {
    gdn::DecodeArgs d;
    gdn_status st = check_decode(cfg, B_max, T, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool,
                                 pool_slots, slots, out_bf16, out_f32, err_flag, workspace, &d);
    if (st != GDN_OK || B_max == 0) return st;
    if (!B_dev) return GDN_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)B_dev & 3u) != 0) return GDN_ERR_MISALIGNED;
    d.B_dev = B_dev;
    return from_cuda(gdn::launch_decode_fused(d, (cudaStream_t)stream));
}

gdn_status gdn_decode_step_varlen(const gdn_config* cfg, int32_t B, const int32_t* cu_seqlens, int32_t T_max,
                                  int32_t total_tokens, const uint16_t* qkv, const uint16_t* a, const uint16_t* b,
                                  const uint16_t* z, const uint16_t* conv_w, const float* A_log,
                                  const float* dt_bias, const uint16_t* norm_w, uint16_t* conv_pool,
                                  float* state_pool, int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                                  float* out_f32, int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if (total_tokens < 0) return GDN_ERR_INVALID_ARGUMENT;
    if ((st = check_batch(B, T_max, pool_slots, sh)) != GDN_OK) return st;
    if (B == 0 || total_tokens == 0) return GDN_OK;  // no sequence has a token: nothing to do
    if (!cu_seqlens) return GDN_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)cu_seqlens & 3u) != 0) return GDN_ERR_MISALIGNED;
    if ((st = check_pointers({conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool, slots}, {out_f32, err_flag})) !=
        GDN_OK)
        return st;
    if ((st = check_pointers({qkv, a, b, z, out_bf16}, {})) != GDN_OK) return st;
    gdn::DecodeArgs d{sh, B, T_max, pool_slots, 1, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool,
                      state_pool, slots, out_bf16, out_f32, err_flag, nullptr, cu_seqlens, total_tokens};
    if (!gdn::multitoken_supported(d)) return GDN_ERR_UNSUPPORTED;
    return from_cuda(gdn::launch_decode_multitoken(d, (cudaStream_t)stream));
}

gdn_status gdn_spec_verify(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv, const uint16_t* a,
                           const uint16_t* b, const uint16_t* z, const uint16_t* conv_w, const float* A_log,
                           const float* dt_bias, const uint16_t* norm_w, const uint16_t* conv_pool,
                           const float* state_pool, int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                           float* out_f32, float* spec_k, float* spec_delta, float* spec_alpha, int32_t* err_flag,
                           void* stream) {
    gdn::DecodeArgs d;
    // the pools are only read in verify mode
    gdn_status st = check_decode(cfg, B, T, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w,
                                 const_cast<uint16_t*>(conv_pool), const_cast<float*>(state_pool), pool_slots, slots,
                                 out_bf16, out_f32, err_flag, nullptr, &d);
    if (st != GDN_OK || B == 0) return st;
    if ((st = check_pointers({spec_k, spec_delta, spec_alpha}, {})) != GDN_OK) return st;
    d.T = T;
    d.spec_k = spec_k;
    d.spec_delta = spec_delta;
    d.spec_alpha = spec_alpha;
    if (!gdn::multitoken_supported(d)) return GDN_ERR_UNSUPPORTED;
    return from_cuda(gdn::launch_decode_multitoken(d, (cudaStream_t)stream));
}

gdn_status gdn_spec_commit(const gdn_config* cfg, int32_t B, int32_t T, const int32_t* n_accept,
                           const uint16_t* qkv, uint16_t* conv_pool, float* state_pool, int32_t pool_slots,
                           const int32_t* slots, const float* spec_k, const float* spec_delta,
                           const float* spec_alpha, int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_batch(B, T, pool_slots, sh)) != GDN_OK) return st;
    if (B == 0) return GDN_OK;
    if ((st = check_pointers({n_accept, qkv, conv_pool, state_pool, slots, spec_k, spec_delta, spec_alpha},
                             {err_flag})) != GDN_OK)
        return st;
    gdn::SpecCommitArgs c{sh, B, T, pool_slots, n_accept, qkv, conv_pool, state_pool, slots,
                          spec_k, spec_delta, spec_alpha, err_flag};
    return from_cuda(gdn::launch_spec_commit(c, (cudaStream_t)stream));
}

gdn_status gdn_in_proj(const gdn_config* cfg, int32_t hidden, int32_t rows, const uint16_t* x,
                       const uint16_t* w_in, uint16_t* qkv, uint16_t* z, uint16_t* a, uint16_t* b, float* out_f32,
                       int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_proj_sizes(hidden, rows)) != GDN_OK) return st;
    if (rows == 0) return GDN_OK;
    if ((st = check_pointers({x, w_in, qkv, z, a, b}, {out_f32, err_flag})) != GDN_OK) return st;
    const int Z = sh.Hv * sh.dv;
    gdn::ProjArgs p{};
    p.N = sh.C + Z + 2 * sh.Hv;
    p.K = hidden;
    p.R = rows;
    p.x = x;
    p.w = w_in;
    p.nseg = 4;
    const int starts[4] = {0, sh.C, sh.C + Z, sh.C + Z + sh.Hv}, widths[4] = {sh.C, Z, sh.Hv, sh.Hv};
    uint16_t* outs[4] = {qkv, z, a, b};
    for (int i = 0; i < 4; ++i) {
        p.seg_start[i] = starts[i];
        p.seg_width[i] = widths[i];
        p.seg_out[i] = outs[i];
    }
    p.out_f32 = out_f32;
    p.err_flag = err_flag;
    return launch_proj(p, (cudaStream_t)stream);
}

gdn_status gdn_out_proj(const gdn_config* cfg, int32_t hidden, int32_t rows, const uint16_t* y,
                        const uint16_t* w_out, uint16_t* out, float* out_f32, int32_t* err_flag, void* stream) {
    gdn::Shape sh;
    gdn_status st = check_config(cfg, &sh);
    if (st != GDN_OK) return st;
    if ((st = check_proj_sizes(hidden, rows)) != GDN_OK) return st;
    if (rows == 0) return GDN_OK;
    if ((st = check_pointers({y, w_out, out}, {out_f32, err_flag})) != GDN_OK) return st;
    gdn::ProjArgs p{};
    p.N = hidden;
    p.K = sh.Hv * sh.dv;
    p.R = rows;
    p.x = y;
    p.w = w_out;
    p.nseg = 1;
    p.seg_start[0] = 0;
    p.seg_width[0] = hidden;
    p.seg_out[0] = out;
    p.out_f32 = out_f32;
    p.err_flag = err_flag;
    return launch_proj(p, (cudaStream_t)stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Scratch for gdn_decode_step_static_scratch: the workspace of gdn_decode_step kept
// in this library's own device memory, so callers that cannot allocate still get the
// dynamic spread of sequences over the SMs. Every GPU that loads the library holds
// this array until the process exits; all calls on a device share it.
namespace {
constexpr size_t kStaticScratchBytes = 256;  // fixed maximum
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = gdn::kMaxDevices;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxScratchDevices];  // device address of g_decode_scratch, per device

// Once per device, with that device current: the array's device address (in host
// code the symbol itself only names a host-side stand-in).
gdn_status static_scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxScratchDevices) return GDN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return GDN_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return GDN_OK;
}
}  // namespace

extern "C" {

gdn_status gdn_decode_step_static_scratch(const gdn_config* cfg, int32_t B, int32_t T, const uint16_t* qkv,
                                          const uint16_t* a, const uint16_t* b, const uint16_t* z,
                                          const uint16_t* conv_w, const float* A_log, const float* dt_bias,
                                          const uint16_t* norm_w, uint16_t* conv_pool, float* state_pool,
                                          int32_t pool_slots, const int32_t* slots, uint16_t* out_bf16,
                                          float* out_f32, int32_t* err_flag, void* stream) {
    const size_t need = gdn_decode_workspace_bytes();
    if (need > kStaticScratchBytes) return GDN_ERR_UNSUPPORTED;  // the fixed array is too small for this build
    // every argument check first: an error return must leave the stream untouched
    gdn::DecodeArgs d;
    gdn_status st = check_decode(cfg, B, T, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, conv_pool, state_pool,
                                 pool_slots, slots, out_bf16, out_f32, err_flag, nullptr, &d);
    if (st != GDN_OK || B == 0) return st;
    void* scratch = nullptr;
    if ((st = static_scratch_address(&scratch)) != GDN_OK) return st;
    d.sched = static_cast<unsigned int*>(scratch);
    // the counters must start at zero; clear them in stream order before the launch
    if (cudaMemsetAsync(scratch, 0, need, (cudaStream_t)stream) != cudaSuccess) return GDN_ERR_CUDA;
    return from_cuda(gdn::launch_decode_fused(d, (cudaStream_t)stream));
}

size_t gdn_decode_static_scratch_bytes(void) { return kStaticScratchBytes; }

gdn_status gdn_selftest_wait_timeout(uint64_t limit_cycles, int32_t* err_flag, uint64_t* cycles, void* stream) {
    if (!err_flag || limit_cycles == 0 || limit_cycles > (1ull << 40)) return GDN_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)err_flag & 3u) != 0 || ((uintptr_t)cycles & 7u) != 0) return GDN_ERR_MISALIGNED;
    return from_cuda(gdn::launch_wait_selftest(limit_cycles, err_flag, reinterpret_cast<unsigned long long*>(cycles),
                                               (cudaStream_t)stream));
}

gdn_status gdn_check_slots_host(const int32_t* slots_host, int32_t B, int32_t pool_slots) {
    if (B < 0 || pool_slots < 0 || (B > 0 && !slots_host)) return GDN_ERR_INVALID_ARGUMENT;
    std::vector<unsigned char> seen((size_t)pool_slots, 0);
    for (int32_t i = 0; i < B; ++i) {
        const int32_t s = slots_host[i];
        if (s < 0 || s >= pool_slots || seen[(size_t)s]) return GDN_ERR_SLOT_RANGE;
        seen[(size_t)s] = 1;
    }
    return GDN_OK;
}

const char* gdn_status_string(gdn_status status) {
    switch (status) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARGUMENT: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape";
        case GDN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case GDN_ERR_SLOT_RANGE: return "slot out of range or repeated";
        case GDN_ERR_CUDA: return "CUDA launch failed";
    }
    return "unknown status";
}

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

}  // extern "C"
