// Backward of the prefill / teacher-forcing chunk-causal attention (training
// form of the chunk mask: hyper.ai summary of the paper, "方法" (teacher
// forcing); the walkthrough's training objective, Fig. 14).
//
// With qr = R q, kr = R k (per-token 3D rotation), S = qr kr^T / sqrt(128) over
// the visible pairs, P = softmax(S) (from the forward's per-row log2 normaliser
// lse), O = P v and the incoming dO:
//   D = rowsum(dO * O),  dP = dO v^T,  dS = P * (dP - D),
//   dv = P^T dO,  dqr = dS kr / sqrt(128),  dkr = dS^T qr / sqrt(128),
//   dq = R^T dqr,  dk = R^T dkr.
// Two kernels recompute S and dP instead of exchanging partial sums:
//   bwd_dq_kernel   one CTA per (batch, head, 128-query tile): over the key tiles
//                   it sees, S = Q K^T and dP = dO V^T on whole 128-key tiles (both
//                   operands K-major in shared memory), dS in registers, written as
//                   bf16 into one of two TMEM buffers, then dQ += dS K with dS read
//                   from TMEM; the next tile's S and dP run while dS is computed;
//   bwd_dkv_kernel  one CTA per (batch, head, 128-key tile): over the query tiles
//                   that see it, S^T = K Q^T and dP^T = V dO^T, P^T and dS^T
//                   written as bf16 over them in TMEM, then dV += P^T dO and
//                   dK += dS^T Q.
// Each has a TMA warp, an MMA warp and eight compute warps: two per TMEM lane
// quarter, one thread per tile row.  In bwd_dkv_kernel a streamed tile is taken in
// two halves of 64 rows with two TMEM buffers (2-stage ring), so that the products
// of one half run while the compute warps turn the other half's scores into bf16
// operands; each of a lane quarter's two warps takes 32 of a half's 64 columns.  Each
// thread writes its bf16 operands over its own fp32 columns, so a half's operand
// occupies columns [0, 16) and [32, 48) of its region (see mma_tmem_a64).  The rotation back (R^T) and the 1/sqrt(128) are applied to the fp32
// accumulators in the epilogue.
#include <algorithm>
#include <vector>

#include "dz_ops.cuh"
#include "dz_ptx.cuh"

namespace dz {

namespace {

constexpr int BT = 128;                            // rows of a query or key tile
constexpr int BTHREADS = 320;                      // warp 0 TMA, 1 MMA, 2-9 compute
constexpr int BCOMPUTE = BTHREADS - 64;            // two warps per TMEM lane quarter
constexpr int BTILE = BT * HEAD_DIM * 2;           // 32 KiB
constexpr int BHALF = BTILE / 2;                   // 64 dims x 128 rows
constexpr int BSM_FIXED0 = 0;                      // resident tile 0 (Q or K)
constexpr int BSM_FIXED1 = BTILE;                  // resident tile 1 (dO or V)
constexpr int BSM_RING = 2 * BTILE;                // 2 stages x 2 tiles
constexpr int BSM_BAR = BSM_RING + 4 * BTILE;
constexpr int BSM_MISC = BSM_BAR + 256;
constexpr int BSM_VEC = BSM_MISC + 64;             // lse and D of 128 queries, 2 buffers
constexpr int BSMEM_BYTES = BSM_VEC + 2 * 2 * BT * 4 + 1024;
static_assert(BSMEM_BYTES <= 232448, "shared memory");

enum {
  BB_FIX = 0,         // resident tiles landed
  BB_FULL = 1,        // [2] ring stage landed
  BB_EMPTY = 3,       // [2] ring stage consumed
  BB_SDP = 5,         // [2] S and dP (or their transposes) of a half in TMEM buffer u
  BB_READY = 7,       // [2] compute warps wrote the half's bf16 operands (128 arrivals)
  BB_ACC = 9,         // accumulators final
  BB_DRAIN = 10,
  BB_COUNT = 11
};
static_assert(BB_COUNT * 8 <= 256, "barrier area");

// Tiles per (batch, head) whose launch order the host can sort (larger calls keep
// the natural order).
constexpr int BWD_ORDER_MAX = 512;

struct __align__(64) BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // rotated q, rotated k, v, dO: (128, H, S, B)
  const float* lse;                      // [B][H][S], log2 domain
  const float* dd;                       // D = rowsum(dO * O), [B][H][S]
  __nv_bfloat16 *dq, *dk, *dv;           // [B][S][H][128]
  RopeTables rope;
  ChunkGeom geom;
  int mode, L, N, S;                     // S tokens per batch item (queries = keys)
  int B, H, n_tiles;
  int period;                            // TF: N*L (noisy tokens sit at clean positions)
  float scale_log2, scale;
  int* status;
  // Launch order: CTAs go out in groups of head_group (batch, head) pairs; inside a
  // group, rank r of the tiles (heaviest first: order_q for the dQ kernel, order_k for
  // dK/dV) for every pair of the group, then rank r + 1.  The pairs of a group share
  // their streamed tiles through L2, and the lightest tiles come last.
  int head_group, use_order;
  uint16_t order_q[BWD_ORDER_MAX], order_k[BWD_ORDER_MAX];
};

// (batch * H + head, tile) of this CTA under the launch order above.
__device__ __forceinline__ void bwd_unit(const BwdParams& p, const uint16_t* order, int& bh,
                                         int& tile) {
  const int BH = p.B * p.H;
  const int G = p.head_group;
  const int per = G * p.n_tiles;
  const int grp = static_cast<int>(blockIdx.x) / per;
  const int g0 = grp * G;
  const int gs = min(G, BH - g0);
  const int rem = static_cast<int>(blockIdx.x) - grp * per;
  const int rank = rem / gs;
  bh = g0 + (rem - rank * gs);
  tile = p.use_order ? static_cast<int>(order[rank]) : rank;
}

// Visible keys of query s: [a0, a1) and [b0, b1).
__host__ __device__ __forceinline__ void q_keys(const BwdParams& p, int s, int& a0, int& a1, int& b0,
                                       int& b1) {
  const int c = s / p.L;
  a0 = 0;
  b0 = b1 = 0;
  if (p.mode == MODE_PREFILL || c < p.N) {
    a1 = (c + 1) * p.L;
  } else {
    a1 = (c - p.N) * p.L;
    b0 = c * p.L;
    b1 = b0 + p.L;
  }
}

// Queries that see key j: [a0, a1) and [b0, b1).
__device__ __forceinline__ void k_queries(const BwdParams& p, int j, int& a0, int& a1, int& b0,
                                          int& b1) {
  const int c = j / p.L;
  b0 = b1 = 0;
  a0 = c * p.L;
  if (p.mode == MODE_PREFILL) {
    a1 = p.S;
  } else if (c < p.N) {
    a1 = p.N * p.L;
    b0 = (p.N + c + 1) * p.L;
    b1 = 2 * p.N * p.L;
  } else {
    a1 = a0 + p.L;
  }
}

// Does any query of tile qt see any key of tile kt?
__host__ __device__ __forceinline__ bool pair_visible(const BwdParams& p, int qt, int kt) {
  const int q0 = qt * BT, q1 = min(q0 + BT, p.S);
  const int k0 = kt * BT, k1 = min(k0 + BT, p.S);
  for (int c = q0 / p.L; c <= (q1 - 1) / p.L; ++c) {
    int a0, a1, b0, b1;
    q_keys(p, c * p.L, a0, a1, b0, b1);
    if ((a0 < k1 && k0 < a1) || (b0 < k1 && k0 < b1)) return true;
  }
  return false;
}



// Rotary position of token s (noisy teacher-forcing tokens take clean positions).
__device__ __forceinline__ void bpos(const BwdParams& p, int s, int& t, int& h, int& w) {
  token_pos(p.geom, p.period > 0 ? s % p.period : s, 0, t, h, w);
}

// fp32 row chunk of 32 gradient features (pairs 16*c .. 16*c + 15) turned back by
// -theta, scaled, rounded to bf16 and stored (16-byte stores).
__device__ __forceinline__ void store_rotated_back(__nv_bfloat16* dst, const uint32_t (&v)[32],
                                                   const RopeTables& r, int c, int t, int h, int w,
                                                   float scale, int* status) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 cs = __ldg(r.tab + rope_index_checked(r, 16 * c + i, t, h, w, status));
    const float x0 = __uint_as_float(v[2 * i]) * scale, x1 = __uint_as_float(v[2 * i + 1]) * scale;
    const float y0 = __fmaf_rn(x0, cs.x, __fmul_rn(x1, cs.y));
    const float y1 = __fmaf_rn(x1, cs.x, -__fmul_rn(x0, cs.y));
    pk[i] = pack_bf16x2(y0, y1);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
}

__device__ __forceinline__ void tile_load(uint8_t* dst, const CUtensorMap* m, uint64_t* bar,
                                          int h, int row, int b) {
  tma_load_4d(dst, m, bar, 0, h, row, b);
  tma_load_4d(dst + BHALF, m, bar, 64, h, row, b);
}

// K-major A and B (SS) product over the 128 head dims: D[128 x N] = A B^T (N set
// by idesc; b_lo may point at a later row of the B tile).
__device__ __forceinline__ void mma_kmajor(uint32_t d, uint32_t a_lo, uint32_t b_lo,
                                           uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < HEAD_DIM / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * BHALF + (kk & 3) * 32) >> 4;
    mma_ss(d, desc_join(a_lo + off), desc_join(b_lo + off), idesc, kk > 0 ? 1u : 0u);
  }
}

// D[128 x 128] (+)= A B with A (bf16, 128 rows x 64 K) in TMEM and B (64 K rows x
// 128 dims) MN-major in shared memory.  A's K columns 0-31 sit at TMEM columns
// [a, a + 16) and 32-63 at [a + 32, a + 48) (one half per compute warp group).
__device__ __forceinline__ void mma_tmem_a64(uint32_t d, uint32_t a, uint32_t b_lo, uint32_t idesc,
                                             bool acc) {
#pragma unroll
  for (int kk = 0; kk < 64 / 16; ++kk)
    mma_ts(d, a + (kk >> 1) * 32 + (kk & 1) * 8, desc_join(b_lo + ((kk * 16 * 128) >> 4)), idesc,
           (acc || kk > 0) ? 1u : 0u);
}

constexpr uint32_t HALF_ROWS_OFF = (64 * 128) >> 4;  // 64 rows of 128 bytes, in 16-byte units

}  // namespace

// ---------------------------------------------------------------------------
// dQ: one CTA per (batch, head, query tile), whole 128-key tiles.  TMEM: S
// [0,128), dP [128,256), dQ [256,384), dS (bf16) in two buffers [384,448) and
// [448,512).  Shared memory: Q and dO resident, K tiles in a 3-stage ring (a K
// tile is read by S and, a tile later, by dQ), V tiles in a 2-stage ring (read by
// dP only).  Per key tile t the MMA warp issues S(t) and dP(t) as soon as the
// compute warps hold S(t-1) and dP(t-1) in registers, then dQ += dS(t-1) K(t-1)
// once they have written dS(t-1); so the products of tile t run while the compute
// warps turn tile t-1's scores into dS.
// ---------------------------------------------------------------------------
constexpr int DQ_KSTAGES = 3, DQ_VSTAGES = 2;
constexpr int DQ_SM_Q = 0, DQ_SM_DO = BTILE;
constexpr int DQ_SM_K = 2 * BTILE;
constexpr int DQ_SM_V = DQ_SM_K + DQ_KSTAGES * BTILE;
constexpr int DQ_SM_BAR = DQ_SM_V + DQ_VSTAGES * BTILE;
constexpr int DQ_SM_MISC = DQ_SM_BAR + 256;
constexpr int DQ_SMEM_BYTES = DQ_SM_MISC + 64 + 1024;
static_assert(DQ_SMEM_BYTES <= 232448, "shared memory");
enum {
  DQ_FIX = 0,                            // Q and dO landed
  DQ_KFULL = 1,                          // [3] K stage landed
  DQ_KEMPTY = DQ_KFULL + DQ_KSTAGES,     // [3] K stage read by S and dQ
  DQ_VFULL = DQ_KEMPTY + DQ_KSTAGES,     // [2] V stage landed
  DQ_VEMPTY = DQ_VFULL + DQ_VSTAGES,     // [2] V stage read by dP
  DQ_SDP = DQ_VEMPTY + DQ_VSTAGES,       // S and dP of the tile in TMEM
  DQ_READ = DQ_SDP + 1,                  // compute warps hold S, dP in registers (256)
  DQ_DS = DQ_READ + 1,                   // [2] dS written into buffer u (256)
  DQ_DSFREE = DQ_DS + 2,                 // [2] dQ product done reading buffer u
  DQ_ACC = DQ_DSFREE + 2,
  DQ_DRAIN = DQ_ACC + 1,
  DQ_COUNT = DQ_DRAIN + 1
};
static_assert(DQ_COUNT * 8 <= 256, "barrier area");

__global__ void __launch_bounds__(BTHREADS, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + DQ_SM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + DQ_SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + DQ_SM_MISC + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int bh, qt;
  bwd_unit(p, p.order_q, bh, qt);
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int q0 = qt * BT;

  if (tid == 0) {
    mbar_init(&bar[DQ_FIX], 1);
    for (int s = 0; s < DQ_KSTAGES; ++s) {
      mbar_init(&bar[DQ_KFULL + s], 1);
      mbar_init(&bar[DQ_KEMPTY + s], 1);
    }
    for (int s = 0; s < DQ_VSTAGES; ++s) {
      mbar_init(&bar[DQ_VFULL + s], 1);
      mbar_init(&bar[DQ_VEMPTY + s], 1);
    }
    mbar_init(&bar[DQ_SDP], 1);
    mbar_init(&bar[DQ_READ], BCOMPUTE);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bar[DQ_DS + u], BCOMPUTE);
      mbar_init(&bar[DQ_DSFREE + u], 1);
    }
    mbar_init(&bar[DQ_ACC], 1);
    mbar_init(&bar[DQ_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
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
    if (lane == 0) {
      mbar_expect_tx(&bar[DQ_FIX], 2 * BTILE);
      tile_load(smem + DQ_SM_Q, &p.tm_q, &bar[DQ_FIX], h, q0, b);
      tile_load(smem + DQ_SM_DO, &p.tm_do, &bar[DQ_FIX], h, q0, b);
      uint32_t nk = 0, nv = 0;  // K and V tiles issued
      for (int kt = 0; kt < p.n_tiles; ++kt) {
        if (!pair_visible(p, qt, kt)) continue;
        const int ks = nk % DQ_KSTAGES, vs = nv % DQ_VSTAGES;
        if (!mbar_wait(&bar[DQ_KEMPTY + ks], ((nk / DQ_KSTAGES) & 1) ^ 1, abort_flag, p.status)) break;
        mbar_expect_tx(&bar[DQ_KFULL + ks], BTILE);
        tile_load(smem + DQ_SM_K + ks * BTILE, &p.tm_k, &bar[DQ_KFULL + ks], h, kt * BT, b);
        ++nk;
        if (!mbar_wait(&bar[DQ_VEMPTY + vs], ((nv / DQ_VSTAGES) & 1) ^ 1, abort_flag, p.status)) break;
        mbar_expect_tx(&bar[DQ_VFULL + vs], BTILE);
        tile_load(smem + DQ_SM_V + vs * BTILE, &p.tm_v, &bar[DQ_VFULL + vs], h, kt * BT, b);
        ++nv;
      }
      // every issued copy has landed before the CTA exits
      mbar_drain(&bar[DQ_FIX], 0);
      for (uint32_t j = (nk > DQ_KSTAGES ? nk - DQ_KSTAGES : 0); j < nk; ++j)
        mbar_drain(&bar[DQ_KFULL + j % DQ_KSTAGES], (j / DQ_KSTAGES) & 1);
      for (uint32_t j = (nv > DQ_VSTAGES ? nv - DQ_VSTAGES : 0); j < nv; ++j)
        mbar_drain(&bar[DQ_VFULL + j % DQ_VSTAGES], (j / DQ_VSTAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(BT, BT, false);
      const uint32_t id_mn = idesc_bf16(BT, HEAD_DIM, true);
      const uint32_t q_lo = desc_lo(smem_u32(smem + DQ_SM_Q), 16);
      const uint32_t do_lo = desc_lo(smem_u32(smem + DQ_SM_DO), 16);
      bool ok = mbar_wait(&bar[DQ_FIX], 0, abort_flag, p.status);
      tc_fence_after();
      // dQ += dS(t) K(t): A = dS (bf16 pairs in TMEM), B = K tile MN-major (dims
      // contiguous; the two 64-dim halves LBO apart)
      auto issue_dq = [&](uint32_t tt) -> bool {
        const int u = tt & 1, ks = tt % DQ_KSTAGES;
        if (!mbar_wait(&bar[DQ_DS + u], (tt >> 1) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t k_mn = desc_lo(smem_u32(smem + DQ_SM_K + ks * BTILE), BHALF);
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          mma_ts(tmem + 256, tmem + 384 + 64 * u + kk * 8, desc_join(k_mn + ((kk * 16 * 128) >> 4)),
                 id_mn, (tt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar[DQ_DSFREE + u]);
        mma_commit(&bar[DQ_KEMPTY + ks]);
        return true;
      };
      uint32_t t = 0;  // visible key tiles so far
      for (int kt = 0; ok && kt < p.n_tiles; ++kt) {
        if (!pair_visible(p, qt, kt)) continue;
        const int ks = t % DQ_KSTAGES, vs = t % DQ_VSTAGES;
        if (!mbar_wait(&bar[DQ_KFULL + ks], (t / DQ_KSTAGES) & 1, abort_flag, p.status) ||
            !mbar_wait(&bar[DQ_VFULL + vs], (t / DQ_VSTAGES) & 1, abort_flag, p.status) ||
            (t > 0 && !mbar_wait(&bar[DQ_READ], (t - 1) & 1, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_kmajor(tmem, q_lo, desc_lo(smem_u32(smem + DQ_SM_K + ks * BTILE), 16), id_qk);          // S
        mma_kmajor(tmem + 128, do_lo, desc_lo(smem_u32(smem + DQ_SM_V + vs * BTILE), 16), id_qk);  // dP
        mma_commit(&bar[DQ_SDP]);
        mma_commit(&bar[DQ_VEMPTY + vs]);
        if (t > 0 && !issue_dq(t - 1)) {
          ok = false;
          break;
        }
        ++t;
      }
      if (ok && t > 0) ok = issue_dq(t - 1);
      mma_commit(&bar[DQ_ACC]);
      mma_commit(&bar[DQ_DRAIN]);
      mbar_drain(&bar[DQ_DRAIN], 0);
    }
  } else {
    const int quarter = warp & 3;
    const int cg = (warp - 2) >> 2;  // column group: key columns [64 cg, 64 cg + 64) of a tile
    const int r = 32 * quarter + lane;
    const uint32_t la = static_cast<uint32_t>(32 * quarter) << 16;
    const int s = q0 + r;
    const bool valid = s < p.S;
    const int s_eff = valid ? s : p.S - 1;
    size_t vec = static_cast<size_t>(bh) * p.S + s_eff;
    if (!in_bounds(static_cast<long long>(vec), static_cast<long long>(p.B) * p.H * p.S, p.status))
      vec = 0;
    const float lse2 = p.lse[vec];
    const float dsum = p.dd[vec];
    int a0, a1, b0, b1;
    q_keys(p, s_eff, a0, a1, b0, b1);
    uint32_t it = 0;  // visible key tiles so far
    bool ok = true;
    for (int kt = 0; ok && kt < p.n_tiles; ++kt) {
      if (!pair_visible(p, qt, kt)) continue;
      if (!mbar_wait(&bar[DQ_SDP], it & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[64], dp[64];
      {
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(sv + 32);
        uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(dp);
        uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(dp + 32);
        tmem_ld32(tmem + la + 64 * cg, s0);
        tmem_ld32(tmem + la + 64 * cg + 32, s1);
        tmem_ld32(tmem + la + 128 + 64 * cg, d0);
        tmem_ld32(tmem + la + 128 + 64 * cg + 32, d1);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar[DQ_READ]);  // S and dP of this tile may now be overwritten
      const int col0 = kt * BT + 64 * cg;
      uint32_t pk[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int c0 = col0 + 32 * hh;
        const uint32_t keep = range_bits(a0 - c0, a1 - c0) | range_bits(b0 - c0, b1 - c0);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 2 * i + e;
            const float pe = ex2(__uint_as_float(sv[32 * hh + j]) * p.scale_log2 - lse2);
            d2[e] = ((keep >> j) & 1u) ? pe * (__uint_as_float(dp[32 * hh + j]) - dsum) : 0.f;
          }
          pk[16 * hh + i] = pack_bf16x2(d2[0], d2[1]);
        }
      }
      const int u = it & 1;
      // buffer u is free once the dQ product of tile it - 2 has read it
      if (it >= 2 && !mbar_wait(&bar[DQ_DSFREE + u], ((it - 2) >> 1) & 1, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32(tmem + la + 384 + 64 * u + 32 * cg, pk);  // dS, keys [64 cg, 64 cg + 64)
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[DQ_DS + u]);
      ++it;
    }
    if (ok && mbar_wait(&bar[DQ_ACC], 0, abort_flag, p.status)) {
      tc_fence_after();
      int t, hh, w;
      bpos(p, s_eff, t, hh, w);
      const long long dqi = (static_cast<long long>(b * p.S + s_eff) * p.H + h) * HEAD_DIM;
      const bool dq_ok =
          in_bounds(dqi + HEAD_DIM - 1, static_cast<long long>(p.B) * p.S * p.H * HEAD_DIM, p.status);
      __nv_bfloat16* dst = p.dq + dqi;
#pragma unroll 1
      for (int c = 2 * cg; c < 2 * cg + 2; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + la + 256 + 32 * c, v);
        tmem_wait_ld();
        if (it == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (valid && dq_ok) store_rotated_back(dst + 32 * c, v, p.rope, c, t, hh, w, p.scale, p.status);
      }
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

// ---------------------------------------------------------------------------
// dK, dV: one CTA per (batch, head, key tile).  TMEM: S^T [0,128) (P^T bf16 over
// its first 64 columns), dP^T [128,256) (dS^T bf16 over its first 64 columns),
// dV [256,384), dK [384,512).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(BTHREADS, 1) bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + BSM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BSM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + BSM_MISC + 4);
  float* sm_vec = reinterpret_cast<float*>(smem + BSM_VEC);  // [2 buffers][lse 128 | D 128]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int bh, kt;
  bwd_unit(p, p.order_k, bh, kt);
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int k0 = kt * BT;

  if (tid == 0) {
    mbar_init(&bar[BB_FIX], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[BB_FULL + s], 1);
      mbar_init(&bar[BB_EMPTY + s], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bar[BB_SDP + u], 1);
      mbar_init(&bar[BB_READY + u], BCOMPUTE);
    }
    mbar_init(&bar[BB_ACC], 1);
    mbar_init(&bar[BB_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
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
    if (lane == 0) {
      mbar_expect_tx(&bar[BB_FIX], 2 * BTILE);
      tile_load(smem + BSM_FIXED0, &p.tm_k, &bar[BB_FIX], h, k0, b);
      tile_load(smem + BSM_FIXED1, &p.tm_v, &bar[BB_FIX], h, k0, b);
      uint32_t it = 0;
      for (int qt = 0; qt < p.n_tiles; ++qt) {
        if (!pair_visible(p, qt, kt)) continue;
        const int st = it & 1;
        if (!mbar_wait(&bar[BB_EMPTY + st], ((it >> 1) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* ring = smem + BSM_RING + st * 2 * BTILE;
        mbar_expect_tx(&bar[BB_FULL + st], 2 * BTILE);
        tile_load(ring, &p.tm_q, &bar[BB_FULL + st], h, qt * BT, b);
        tile_load(ring + BTILE, &p.tm_do, &bar[BB_FULL + st], h, qt * BT, b);
        ++it;
      }
      mbar_drain(&bar[BB_FIX], 0);
      for (uint32_t j = (it > 2 ? it - 2 : 0); j < it; ++j) mbar_drain(&bar[BB_FULL + (j & 1)], (j >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_n64 = idesc_bf16(BT, 64, false);
      const uint32_t id_mn = idesc_bf16(BT, HEAD_DIM, true);
      const uint32_t k_lo = desc_lo(smem_u32(smem + BSM_FIXED0), 16);
      const uint32_t v_lo = desc_lo(smem_u32(smem + BSM_FIXED1), 16);
      bool ok = mbar_wait(&bar[BB_FIX], 0, abort_flag, p.status);
      tc_fence_after();
      // half-step j = 2 * (query tile ordinal) + half; TMEM buffer = half
      auto grads = [&](uint32_t jj) {
        const int hf = jj & 1, st = (jj >> 1) & 1;
        const uint32_t q_mn = desc_lo(smem_u32(smem + BSM_RING + st * 2 * BTILE), BHALF);
        const uint32_t do_mn = desc_lo(smem_u32(smem + BSM_RING + st * 2 * BTILE + BTILE), BHALF);
        mma_tmem_a64(tmem + 256, tmem + 128 * hf, do_mn + hf * HALF_ROWS_OFF, id_mn, jj > 0);      // dV += P^T dO
        mma_tmem_a64(tmem + 384, tmem + 128 * hf + 64, q_mn + hf * HALF_ROWS_OFF, id_mn, jj > 0);  // dK += dS^T Q
        if (hf == 1) mma_commit(&bar[BB_EMPTY + st]);
      };
      uint32_t t = 0;
      for (int qt = 0; ok && qt < p.n_tiles; ++qt) {
        if (!pair_visible(p, qt, kt)) continue;
        const int st = t & 1;
        const uint32_t q_lo = desc_lo(smem_u32(smem + BSM_RING + st * 2 * BTILE), 16);
        const uint32_t do_lo = desc_lo(smem_u32(smem + BSM_RING + st * 2 * BTILE + BTILE), 16);
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t jj = 2 * t + hf;
          if (jj >= 2) {
            if (!mbar_wait(&bar[BB_READY + hf], ((jj - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            grads(jj - 2);
          }
          if (hf == 0) {
            if (!mbar_wait(&bar[BB_FULL + st], (t >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
          }
          mma_kmajor(tmem + 128 * hf, k_lo, q_lo + hf * HALF_ROWS_OFF, id_n64);        // S^T
          mma_kmajor(tmem + 128 * hf + 64, v_lo, do_lo + hf * HALF_ROWS_OFF, id_n64);  // dP^T
          mma_commit(&bar[BB_SDP + hf]);
        }
        ++t;
      }
      for (uint32_t jj = (2 * t >= 2 ? 2 * t - 2 : 0); ok && jj < 2 * t; ++jj) {
        if (!mbar_wait(&bar[BB_READY + (jj & 1)], (jj >> 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        grads(jj);
      }
      mma_commit(&bar[BB_ACC]);
      mma_commit(&bar[BB_DRAIN]);
      mbar_drain(&bar[BB_DRAIN], 0);
    }
  } else {
    const int quarter = warp & 3;
    const int cg = (warp - 2) >> 2;  // column group: columns [32 cg, 32 cg + 32) of a half
    const int r = 32 * quarter + lane;
    const int ct = tid - 64;         // 0..255 among the compute threads
    const uint32_t la = static_cast<uint32_t>(32 * quarter) << 16;
    const int j = k0 + r;
    const bool valid = j < p.S;
    const int j_eff = valid ? j : p.S - 1;
    int a0, a1, b0, b1;
    k_queries(p, j_eff, a0, a1, b0, b1);
    const size_t vbase = static_cast<size_t>(bh) * p.S;
    uint32_t it = 0;  // visible query tiles so far
    bool ok = true;
    for (int qt = 0; ok && qt < p.n_tiles; ++qt) {
      if (!pair_visible(p, qt, kt)) continue;
      const int q0 = qt * BT;
      // the query tile's lse (threads 0-127) and D (128-255), double-buffered across tiles
      float* vb = sm_vec + (it & 1) * 2 * BT;
      {
        const int qq = q0 + (ct & (BT - 1));
        const bool vin = qq < p.S && in_bounds(static_cast<long long>(vbase) + qq,
                                               static_cast<long long>(p.B) * p.H * p.S, p.status);
        vb[ct] = vin ? (ct < BT ? p.lse[vbase + qq] : p.dd[vbase + qq]) : 0.f;
      }
      named_bar_sync(1, BCOMPUTE);
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t hs = 2 * it + hf;  // half-step
        if (!mbar_wait(&bar[BB_SDP + hf], (hs >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t col = 128 * hf + 32 * cg;
        uint32_t sv[32], dp[32];
        tmem_ld32(tmem + la + col, sv);
        tmem_ld32(tmem + la + col + 64, dp);
        tmem_wait_ld();
        const int qc = 64 * hf + 32 * cg;  // query column of sv[0] within the tile
        const uint32_t keep = range_bits(a0 - q0 - qc, a1 - q0 - qc) | range_bits(b0 - q0 - qc, b1 - q0 - qc);
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float pr[2], d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int jj = 2 * i + e;
            const float pe = ex2(__uint_as_float(sv[jj]) * p.scale_log2 - vb[qc + jj]);
            pr[e] = ((keep >> jj) & 1u) ? pe : 0.f;
            d2[e] = pr[e] * (__uint_as_float(dp[jj]) - vb[BT + qc + jj]);
          }
          pp[i] = pack_bf16x2(pr[0], pr[1]);
          pd[i] = pack_bf16x2(d2[0], d2[1]);
        }
        tmem_st16(tmem + la + col, pp);       // P^T over this thread's own S^T columns
        tmem_st16(tmem + la + col + 64, pd);  // dS^T over its own dP^T columns
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[BB_READY + hf]);
      }
      ++it;
    }
    if (ok && mbar_wait(&bar[BB_ACC], 0, abort_flag, p.status)) {
      tc_fence_after();
      const size_t row = (static_cast<size_t>(b * p.S + j_eff) * p.H + h) * HEAD_DIM;
      const bool row_ok = in_bounds(static_cast<long long>(row) + HEAD_DIM - 1,
                                    static_cast<long long>(p.B) * p.S * p.H * HEAD_DIM, p.status);
      if (cg == 0) {  // dV
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + la + 256 + 32 * c, v);
          tmem_wait_ld();
          if (it == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (valid && row_ok) {
            uint4* d = reinterpret_cast<uint4*>(p.dv + row + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d[e] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
          }
        }
      } else {  // dK, turned back
        int t, hh, w;
        bpos(p, j_eff, t, hh, w);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + la + 384 + 32 * c, v);
          tmem_wait_ld();
          if (it == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (valid && row_ok)
            store_rotated_back(p.dk + row + 32 * c, v, p.rope, c, t, hh, w, p.scale, p.status);
        }
      }
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

// D = rowsum(dO * O) per (batch, token, head) row, fp32, into [B][H][S].
__global__ void bwd_rowdot_kernel(const uint4* dout, const uint4* out, float* dd, int B, int S,
                                  int H) {
  const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= static_cast<long long>(B) * S * H) return;
  const uint4* a = dout + row * (HEAD_DIM / 8);
  const uint4* c = out + row * (HEAD_DIM / 8);
  float acc = 0.f;
#pragma unroll 4
  for (int i = 0; i < HEAD_DIM / 8; ++i) {
    const uint4 x = a[i], y = c[i];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 xa = *reinterpret_cast<const __nv_bfloat162*>(&xs[k]);
      const __nv_bfloat162 ya = *reinterpret_cast<const __nv_bfloat162*>(&ys[k]);
      acc = __fmaf_rn(__low2float(xa), __low2float(ya), acc);
      acc = __fmaf_rn(__high2float(xa), __high2float(ya), acc);
    }
  }
  const long long h = row % H;
  const long long bs = row / H;
  const long long b = bs / S, s = bs - b * S;
  dd[(b * H + h) * S + s] = acc;
}

cudaError_t launch_backward(const BwdLaunch& a, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DQ_SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BSMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const long long rows = static_cast<long long>(a.B) * a.S * a.H;
  bwd_rowdot_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(
      static_cast<const uint4*>(a.dout), static_cast<const uint4*>(a.out), a.dd, a.B, a.S, a.H);
  BwdParams p;
  p.tm_q = a.tm_q;
  p.tm_k = a.tm_k;
  p.tm_v = a.tm_v;
  p.tm_do = a.tm_do;
  p.lse = a.lse;
  p.dd = a.dd;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.rope = a.rope;
  p.geom = a.geom;
  p.mode = a.mode;
  p.L = a.geom.L;
  p.N = a.N;
  p.S = a.S;
  p.B = a.B;
  p.H = a.H;
  p.n_tiles = (a.S + BT - 1) / BT;
  p.period = a.mode == MODE_TEACHER_FORCING ? a.N * a.geom.L : 0;
  p.scale = 1.f / sqrtf(static_cast<float>(HEAD_DIM));
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HEAD_DIM));
  p.status = a.status;
  // launch order: heaviest tiles first inside groups of (batch, head) pairs whose
  // streamed tiles (2 x S x 256 bytes per pair) fill about a third of the L2
  const long long pair_bytes = 2LL * a.S * HEAD_DIM * 2;
  const long long g = (40LL << 20) / (pair_bytes > 0 ? pair_bytes : 1);
  p.head_group = static_cast<int>(g < 1 ? 1 : (g > a.B * a.H ? a.B * a.H : g));
  p.use_order = p.n_tiles <= BWD_ORDER_MAX ? 1 : 0;
  if (p.use_order) {
    std::vector<int> nq(p.n_tiles, 0), nk(p.n_tiles, 0);
    for (int qt = 0; qt < p.n_tiles; ++qt)
      for (int kt = 0; kt < p.n_tiles; ++kt)
        if (pair_visible(p, qt, kt)) {
          ++nq[qt];
          ++nk[kt];
        }
    std::vector<int> oq(p.n_tiles), ok(p.n_tiles);
    for (int t = 0; t < p.n_tiles; ++t) oq[t] = ok[t] = t;
    std::stable_sort(oq.begin(), oq.end(), [&](int x, int y) { return nq[x] > nq[y]; });
    std::stable_sort(ok.begin(), ok.end(), [&](int x, int y) { return nk[x] > nk[y]; });
    for (int t = 0; t < p.n_tiles; ++t) {
      p.order_q[t] = static_cast<uint16_t>(oq[t]);
      p.order_k[t] = static_cast<uint16_t>(ok[t]);
    }
  }
  const unsigned grid = static_cast<unsigned>(a.B * a.H * p.n_tiles);
  bwd_dq_kernel<<<grid, BTHREADS, DQ_SMEM_BYTES, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkv_kernel<<<grid, BTHREADS, BSMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dz
