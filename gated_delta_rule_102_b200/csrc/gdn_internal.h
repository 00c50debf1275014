// Internal interface between the C-ABI layer (argument checks) and the kernel
// launchers. Nothing here is exported.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Devices a process may use with this library (per-device host caches are this large).
constexpr int kMaxDevices = 64;

struct Shape {
    int Hk, Hv, dk, dv, W;  // heads, head dims, conv width
    int C;                  // 2*Hk*dk + Hv*dv
    float l2_eps, rms_eps, q_scale;
};

struct DecodeArgs {
    Shape sh;
    int B, T, P;
    int NS;  // column slices per v-head (dv / NS columns per CTA)
    const uint16_t* qkv;
    const uint16_t* a;
    const uint16_t* b;
    const uint16_t* z;
    const uint16_t* conv_w;
    const float* A_log;
    const float* dt_bias;
    const uint16_t* norm_w;
    uint16_t* conv_pool;
    float* state_pool;
    const int32_t* slots;
    uint16_t* out;
    float* out_f32;
    int32_t* err_flag;
    unsigned int* sched;  // nullable: two zeroed counters for the dynamic schedule of the persistent kernel
    // nullable: [B+1] device offsets of each sequence's tokens in the packed inputs and
    // outputs (sequence i has the rows cu_seqlens[i] .. cu_seqlens[i+1]-1, at most T of
    // them); null: every sequence has T tokens, sequence i at rows i*T ..
    const int32_t* cu_seqlens;
    int32_t total_rows;  // with cu_seqlens: rows of the packed tensors (a sequence's rows must lie inside)
    // speculative verify (all three set, multi-token kernel only): the pools are not
    // written; per token the normalised key [rows][Hk][dk], the write delta
    // [rows][Hv][dv] and the decay [rows][Hv] are
    float* spec_k;
    float* spec_delta;
    float* spec_alpha;
    // nullable: device int32 holding this launch's batch count (0..B); B then only
    // bounds it and sizes the launch, so one captured launch serves any smaller batch
    const int32_t* B_dev;
};

// Commit of the accepted prefix of a speculative verify call.
struct SpecCommitArgs {
    Shape sh;
    int B, T, P;
    const int32_t* n_accept;
    const uint16_t* qkv;
    uint16_t* conv_pool;
    float* state_pool;
    const int32_t* slots;
    const float* spec_k;
    const float* spec_delta;
    const float* spec_alpha;
    int32_t* err_flag;
};

struct ConvArgs {
    Shape sh;
    int B, T, P;
    const uint16_t* qkv;
    const uint16_t* conv_w;
    uint16_t* conv_pool;
    const int32_t* slots;
    float* q;
    float* k;
    float* v;
    int32_t* err_flag;
};

struct RecurrentArgs {
    Shape sh;
    int B, T, P;
    int NS;
    const float* q;
    const float* k;
    const float* v;
    const uint16_t* a;
    const uint16_t* b;
    const float* A_log;
    const float* dt_bias;
    float* state_pool;
    const int32_t* slots;
    float* o;
    int32_t* err_flag;
};

struct NormArgs {
    Shape sh;
    int rows;
    const float* o;
    const uint16_t* z;
    const uint16_t* norm_w;
    uint16_t* out;
    float* out_f32;
};

// The projection GEMM D = X W^T (bf16 in, fp32 accumulate, bf16 out): X [R][K] token
// rows, W [N][K] weight rows; output features are routed to up to four row-major
// outputs by consecutive ranges (segment i holds features seg_start[i] ..
// seg_start[i] + seg_width[i] - 1 as [R][seg_width[i]]).
constexpr int kProjMaxRows = 256;
struct ProjArgs {
    int N, K, R;
    int slices;  // K-slices per weight tile (the cluster size)
    const uint16_t* x;
    const uint16_t* w;
    int nseg;
    int seg_start[4];
    int seg_width[4];
    uint16_t* seg_out[4];
    float* out_f32;  // nullable: [R][N] fp32 before rounding
    int32_t* err_flag;
};
// K-slices per weight tile (the cluster size) for a launch; the first call per shape
// queries the device (sets the kernel attribute, occupancy), later ones hit a cache.
cudaError_t proj_slices(int N, int K, int R, int* slices);
int proj_smem_bytes(int R);
cudaError_t launch_proj_gemm(const ProjArgs& a, cudaStream_t stream);

// Column slices per v-head for the fused kernel: the cluster of one (sequence,
// k-head) holds G * NS CTAs, at most 8.
int decode_column_splits(int B, int Hv, int G, int dv);
// Column slices per v-head for the stand-alone recurrence (no cluster).
int recurrent_column_splits(int B, int Hv, int dv);

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t stream);
// Persistent single-token kernel: whether it handles the shape, its co-resident
// cluster capacity, and the launch.
bool persistent_supported(const DecodeArgs& a);
cudaError_t persistent_capacity(const DecodeArgs& a, int* max_clusters);
cudaError_t launch_decode_persistent(const DecodeArgs& a, cudaStream_t stream);
// Multi-token kernel (state in registers across the launch's tokens); for dk = dv = 128
// it hands the launch to the chunked tensor-core kernel.
bool multitoken_supported(const DecodeArgs& a);
cudaError_t launch_decode_multitoken(const DecodeArgs& a, cudaStream_t stream);
bool chunk_supported(const DecodeArgs& a);
cudaError_t launch_decode_chunk(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_spec_commit(const SpecCommitArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint64_t limit_cycles, int32_t* err_flag, unsigned long long* cycles,
                                 cudaStream_t stream);
cudaError_t launch_conv_update(const ConvArgs& a, cudaStream_t stream);
cudaError_t launch_recurrent(const RecurrentArgs& a, cudaStream_t stream);
cudaError_t launch_gated_rmsnorm(const NormArgs& a, cudaStream_t stream);

}  // namespace gdn
