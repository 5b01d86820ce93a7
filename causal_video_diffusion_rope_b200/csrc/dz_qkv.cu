// QKV projection of a run of chunk tokens with the 3D rotary embedding and the
// KV-cache append fused into the GEMM epilogue.
//
// y = x W^T for x bf16 [M][K] (M = B*S tokens, K = d_model) and W bf16 [N][K]
// (N = 3*H*128 output features: q, then k, then v, each head's 128 features
// contiguous).  The q and k features of every token are turned by the token's
// (t, h, w) rotation in fp32 straight from the fp32 accumulator, then every
// output is rounded once to bf16 and written as q, k, v [M][H][128]; with a
// cache, k and v also go to cache rows [row0, row0 + S) of their batch item.
// The projection is the causal self-attention's input step in the DiT block
// ("DreamZero (WAM) 模型架构", §2.3 block diagram: RMSNorm, modulation, causal
// self-attention with RoPE on the latent sequence).
//
// One persistent CTA per SM walks output tiles of 256 tokens x BN features,
// n-tile major so that the CTAs working at one time share the same weight tile
// through L2.  BN (a multiple of 16, at most 256) is chosen per call so that the
// tiles fill the SMs in as few waves as possible (for one 464-token chunk of the
// 40-head DiT, BN = 208 gives 2 x 74 = 148 tiles, one per SM).  A tile is two
// 128-row halves that share each weight slice, so every byte brought to the SM
// feeds twice the products of a 128 x BN tile.  Warp 0 issues TMA loads of
// 64-wide K slices into a 3-stage ring, warp 1 allocates TMEM and issues
// tcgen05.mma (M=128, N=BN, K=16, both operands K-major SW128 in shared memory;
// two per K step, one per half) into two TMEM accumulators, and warps 2-9 (one
// per TMEM lane quarter and half) drain them 16 features at a time (rotation,
// bf16 rounding, stores).
#include "dz_ops.cuh"
#include "dz_ptx.cuh"

namespace dz {

namespace {

constexpr int QBM = 256, QBN = 256, QBK = 64, QSTAGES = 3;
constexpr int QPREFETCH = 8;             // weight K slices requested into L2 ahead of their load
constexpr int QHALF = 128;               // rows per MMA (one TMEM lane each)
constexpr int QTHREADS = 320;            // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int QA_BYTES = QBM * QBK * 2;  // 32 KiB
constexpr int QB_BYTES = QBN * QBK * 2;  // 32 KiB
constexpr int QSTAGE_BYTES = QA_BYTES + QB_BYTES;
constexpr int QSM_BAR = QSTAGES * QSTAGE_BYTES;
constexpr int QSM_MISC = QSM_BAR + 256;
constexpr int QSM_ROPE = QSM_MISC + 64;             // staged rotary rows of the call
constexpr int QSMEM_BYTES = QSM_ROPE + QKV_ROPE_STAGE_MAX * 8 + 1024;  // + alignment slack
static_assert(QSMEM_BYTES <= 232448, "shared memory");

enum {
  QB_FULL = 0,
  QB_EMPTY = QB_FULL + QSTAGES,
  QB_ACC_FULL = QB_EMPTY + QSTAGES,
  QB_ACC_EMPTY = QB_ACC_FULL + 1,
  QB_DRAIN = QB_ACC_EMPTY + 1,
  QB_COUNT = QB_DRAIN + 1
};
static_assert(QB_COUNT * 8 <= 256, "barrier area");

struct __align__(64) QkvParams {
  CUtensorMap tm_x, tm_w;
  __nv_bfloat16 *q, *k, *v;
  __nv_bfloat16 *ck, *cv;  // cache (null: no append)
  int cache_cap, cache_row0;
  int M, S, H, K, N;
  int cache_batch;  // batch items of the cache (bounds-checked build)
  int bn;  // features per tile
  int m_tiles, n_tiles;
  RopeTables rope;
  ChunkGeom geom;
  int first_chunk;
  int stage_ok, stage_t0, stage_nt;
  int* status;
};

// Requests a 2-D tile into L2 (no shared memory, no completion): the later TMA
// load of the same tile then finds it there.
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1)
               : "memory");
}

// 16 B stores of 16 bf16 values (a 32-byte row piece).
__device__ __forceinline__ void store_piece(__nv_bfloat16* dst, const uint32_t (&pk)[8]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}


}  // namespace

__global__ void __launch_bounds__(QTHREADS, 1) qkv_rope_kernel(const __grid_constant__ QkvParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + QSM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + QSM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + QSM_MISC + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = p.m_tiles * p.n_tiles;
  const int KB = p.K / QBK;

  if (tid == 0) {
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&bar[QB_FULL + s], 1);
      mbar_init(&bar[QB_EMPTY + s], 1);
    }
    mbar_init(&bar[QB_ACC_FULL], 1);
    mbar_init(&bar[QB_ACC_EMPTY], 8 * 32);
    mbar_init(&bar[QB_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const int nt = tile / p.m_tiles, mt = tile - nt * p.m_tiles;
        // the weight slices stream from DRAM: ask for them well before the ring has room
        for (int j = QSTAGES; j < QPREFETCH && j < KB; ++j)
          tma_prefetch_l2_2d(&p.tm_w, j * QBK, nt * p.bn);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          if (kb + QPREFETCH < KB) tma_prefetch_l2_2d(&p.tm_w, (kb + QPREFETCH) * QBK, nt * p.bn);
          const int st = it % QSTAGES;
          const uint32_t ph = (it / QSTAGES) & 1;
          if (!mbar_wait(&bar[QB_EMPTY + st], ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* sa = smem + st * QSTAGE_BYTES;
          mbar_expect_tx(&bar[QB_FULL + st], QA_BYTES + p.bn * QBK * 2);
          tma_load_2d(sa, &p.tm_x, &bar[QB_FULL + st], kb * QBK, mt * QBM);
          tma_load_2d(sa + QA_BYTES, &p.tm_w, &bar[QB_FULL + st], kb * QBK, nt * p.bn);
        }
      }
      // every issued copy has landed before the CTA exits
      const uint32_t n_iss = it;
      for (uint32_t j = (n_iss > QSTAGES ? n_iss - QSTAGES : 0); j < n_iss; ++j)
        mbar_drain(&bar[QB_FULL + j % QSTAGES], (j / QSTAGES) & 1);
    }
  } else if (warp == 1) {
    // ---------------- tcgen05 issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(QHALF, p.bn, false);
      const uint32_t base_lo = desc_lo(smem_u32(smem), 16);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++lt) {
        // the epilogue has drained the accumulators (tile lt - 1)
        if (!mbar_wait(&bar[QB_ACC_EMPTY], (lt & 1) ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int st = it % QSTAGES;
          const uint32_t ph = (it / QSTAGES) & 1;
          if (!mbar_wait(&bar[QB_FULL + st], ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = base_lo + ((st * QSTAGE_BYTES) >> 4);
          const uint32_t b0 = a0 + (QA_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < QBK / 16; ++kk) {
            const uint64_t bd = desc_join(b0 + ((kk * 32) >> 4));
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
              mma_ss(tmem + hf * QBN,
                     desc_join(a0 + ((hf * QHALF * QBK * 2 + kk * 32) >> 4)), bd, idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar[QB_EMPTY + st]);
        }
        if (!ok) break;
        mma_commit(&bar[QB_ACC_FULL]);
      }
      mma_commit(&bar[QB_DRAIN]);
      mbar_drain(&bar[QB_DRAIN], 0);
    }
  } else {
    // ---------------- epilogue: warps 2..9, one token row per thread ----------------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = half * QHALF + 32 * quarter + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const int HD = p.H * HEAD_DIM;
    // the call's rotary rows (t in [stage_t0, stage_t0 + stage_nt), every h < gh and
    // w < gw) go to shared memory while the first tile accumulates
    RopeTables rope = p.rope;
    if (p.stage_ok) {
      float2* st_tab = reinterpret_cast<float2*>(smem + QSM_ROPE);
      const int nt_ = p.stage_nt * p.rope.pt, nh = p.geom.gh * p.rope.ph, nw = p.geom.gw * p.rope.pw;
      const float2* gt = p.rope.tab + p.rope.off_t + p.stage_t0 * p.rope.pt;
      const float2* gh = p.rope.tab + p.rope.off_h;
      const float2* gw = p.rope.tab + p.rope.off_w;
      for (int i = tid - 64; i < nt_ + nh + nw; i += QTHREADS - 64) {
        const long long gi = i < nt_ ? p.rope.off_t + static_cast<long long>(p.stage_t0) * p.rope.pt + i
                                     : (i < nt_ + nh ? p.rope.off_h + i - nt_ : p.rope.off_w + i - nt_ - nh);
        if (in_bounds(gi, p.rope.n, p.status))
          st_tab[i] = i < nt_ ? gt[i] : (i < nt_ + nh ? gh[i - nt_] : gw[i - nt_ - nh]);
      }
      named_bar_sync(1, QTHREADS - 64);
      rope.tab = st_tab;
      rope.off_t = -p.stage_t0 * p.rope.pt;
      rope.off_h = nt_;
      rope.off_w = nt_ + nh;
      rope.n = nt_ + nh + nw;
    }
    int lt = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++lt) {
      if (!mbar_wait(&bar[QB_ACC_FULL], lt & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int nt = tile / p.m_tiles, mt = tile - nt * p.m_tiles;
      const int m = mt * QBM + r;
      const bool valid = m < p.M;
      const int bb = valid ? m / p.S : 0;
      const int s = valid ? m - bb * p.S : 0;
      int t = 0, hh = 0, w = 0;
      token_pos(p.geom, s, p.first_chunk, t, hh, w);
      // 16-feature pieces: each lies inside one head (16 divides 128 and BN); piece
      // c + 1 is read from TMEM while piece c is turned and stored
      int pieces = p.bn / 16;
      if (nt * p.bn + pieces * 16 > p.N) pieces = (p.N - nt * p.bn) / 16;
      uint32_t v[16], vn[16];
      tmem_ld16(tmem + lane_addr + half * QBN, v);
      tmem_wait_ld();
#pragma unroll 1
      for (int c = 0; c < pieces; ++c) {
        const int n = nt * p.bn + c * 16;  // feature of column 0 of this piece
        if (c + 1 < pieces) tmem_ld16(tmem + lane_addr + half * QBN + (c + 1) * 16, vn);
        const int sec = n / HD;  // 0 q, 1 k, 2 v
        const int rem = n - sec * HD;
        const int head = rem / HEAD_DIM, d0 = rem - head * HEAD_DIM;
        float2 cs[8];
        if (sec < 2) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            cs[i] = rope.tab[rope_index_checked(rope, d0 / 2 + i, t, hh, w, p.status)];
        }
        uint32_t pk[8];
        if (sec < 2) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
            const float y0 = __fmaf_rn(x0, cs[i].x, -__fmul_rn(x1, cs[i].y));
            const float y1 = __fmaf_rn(x0, cs[i].y, __fmul_rn(x1, cs[i].x));
            pk[i] = pack_bf16x2(y0, y1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        if (valid) {
          const long long oi = (static_cast<long long>(m) * p.H + head) * HEAD_DIM + d0;
          if (in_bounds(oi + 15, static_cast<long long>(p.M) * p.H * HEAD_DIM, p.status))
            store_piece((sec == 0 ? p.q : (sec == 1 ? p.k : p.v)) + oi, pk);
          if (sec > 0 && p.ck) {
            const long long ci =
                ((static_cast<long long>(bb) * p.cache_cap + p.cache_row0 + s) * p.H + head) * HEAD_DIM + d0;
            if (in_bounds(ci + 15,
                          static_cast<long long>(p.cache_batch) * p.cache_cap * p.H * HEAD_DIM,
                          p.status))
              store_piece((sec == 1 ? p.ck : p.cv) + ci, pk);
          }
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = vn[i];
      }
      // this thread's accumulator loads are complete: the MMA warp may reuse them
      tc_fence_before();
      mbar_arrive(&bar[QB_ACC_EMPTY]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

int qkv_tile_n(long long M, long long N, int num_sms) {
  // least work for the busiest SM: waves x (BN + a fixed 32 for the token slice each
  // K step also loads), the larger BN on a tie
  const long long m_tiles = (M + QBM - 1) / QBM;
  int best = QBN;
  long long best_cost = -1;
  for (int bn = QBN; bn >= 64; bn -= 16) {
    const long long tiles = m_tiles * ((N + bn - 1) / bn);
    const long long cost = (tiles + num_sms - 1) / num_sms * (bn + 32);
    if (best_cost < 0 || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

cudaError_t launch_qkv_rope(const QkvLaunch& a, cudaStream_t stream) {
  if (a.bn < 16 || a.bn > QBN || a.bn % 16 != 0) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(
        qkv_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, QSMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  QkvParams p;
  p.tm_x = a.tm_x;
  p.tm_w = a.tm_w;
  p.q = static_cast<__nv_bfloat16*>(a.q);
  p.k = static_cast<__nv_bfloat16*>(a.k);
  p.v = static_cast<__nv_bfloat16*>(a.v);
  p.ck = static_cast<__nv_bfloat16*>(a.ck);
  p.cv = static_cast<__nv_bfloat16*>(a.cv);
  p.cache_cap = a.cache_cap;
  p.cache_row0 = a.cache_row0;
  p.cache_batch = a.cache_batch;
  p.M = a.M;
  p.S = a.S;
  p.H = a.H;
  p.K = a.K;
  p.N = 3 * a.H * HEAD_DIM;
  p.bn = a.bn;
  p.m_tiles = (a.M + QBM - 1) / QBM;
  p.n_tiles = (p.N + p.bn - 1) / p.bn;
  p.rope = a.rope;
  p.geom = a.geom;
  p.first_chunk = a.first_chunk;
  p.stage_ok = a.stage_ok;
  p.stage_t0 = a.stage_t0;
  p.stage_nt = a.stage_nt;
  p.status = a.status;
  const int total = p.m_tiles * p.n_tiles;
  const int grid = total < a.num_sms ? total : a.num_sms;
  qkv_rope_kernel<<<grid, QTHREADS, QSMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dz
