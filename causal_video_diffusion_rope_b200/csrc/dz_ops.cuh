// Launch descriptions of the fused QKV projection (dz_qkv.cu) and the attention
// backward (dz_bwd.cu), shared with the host API (dz_api.cu).
#pragma once
#include "dz_internal.cuh"

namespace dz {

// Fused QKV projection + rotation (+ cache append); see dz_qkv.cu.
struct QkvLaunch {
  CUtensorMap tm_x, tm_w;  // x [M][K], w [3*H*128][K], bf16, 64 x 256 / 64 x bn boxes, SW128
  void *q, *k, *v;         // [M][H][128]
  void *ck, *cv;           // cache or null
  int cache_cap, cache_row0, cache_batch;
  int M, S, H, K;
  int bn;  // output features per tile (qkv_tile_n)
  RopeTables rope;
  ChunkGeom geom;
  int first_chunk;
  int stage_ok, stage_t0, stage_nt;  // rotary rows staged in shared memory (see AttnLaunch)
  int* status;
  int num_sms;
};
// Capacity (float2 entries) of the projection kernel's shared-memory rotary table.
constexpr int QKV_ROPE_STAGE_MAX = 4096;
// Output features per projection tile (a multiple of 16, at most 256) for M tokens
// and N features on num_sms SMs.
int qkv_tile_n(long long M, long long N, int num_sms);
cudaError_t launch_qkv_rope(const QkvLaunch& a, cudaStream_t stream);

// Backward of the prefill / teacher-forcing attention; see dz_bwd.cu.
struct BwdLaunch {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // rotated q, rotated k, v, dO (4-D, 128-row boxes)
  const void *out, *dout;               // bf16 [B][S][H][128]
  const float* lse;                     // [B][H][S] from the forward (log2 domain)
  float* dd;                            // workspace [B][H][S]: rowsum(dO * O)
  void *dq, *dk, *dv;                   // bf16 [B][S][H][128]
  RopeTables rope;
  ChunkGeom geom;
  int mode, N, S, B, H;
  int* status;
};
cudaError_t launch_backward(const BwdLaunch& a, cudaStream_t stream);

}  // namespace dz
