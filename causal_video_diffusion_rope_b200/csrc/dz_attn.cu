// Chunk-causal multi-head attention with fused 3D rotary embedding for sm_100a.
//
// What it computes (see include/dz.h): out = softmax(R q (R k)^T / sqrt(128),
// chunk mask) v per (batch, head) -- the causal self-attention of the Causal
// WAN DiT ("DreamZero (WAM) 模型架构", §2.3) with the chunk-level visibility of
// the paper's method section (a noisy chunk sees the clean context of earlier
// chunks and itself, never future tokens).
//
// Design (one persistent CTA per SM, 384 threads = 12 warps, 1 CTA/SM; 12 warps
// keep 3 warps per SM sub-partition, which leaves up to 168 registers a thread):
//   warp 0        TMA producer: Q tiles of the current unit, then K and V tiles
//                 through a 2-stage ring (128B-swizzled, K-major rows of 128 dims).
//   warp 1        TMEM owner (512 columns) and single-thread tcgen05.mma issuer.
//   warps 2-3     rotary gate: rotates the Q tiles and the call's own K tiles in
//                 shared memory (RoPE fused into the tile load, two rows per
//                 thread), then releases them to the tensor core.  Cache K tiles
//                 pass through unrotated.
//   warps 4-7     softmax group 0 (Q tile 0, one query row per thread)
//   warps 8-11    softmax group 1 (Q tile 1)
// TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512) (fp32 columns); the
// bf16 probabilities P_q overwrite the first 64 columns of S_q and feed the PV
// product directly from TMEM.  The issue order per key tile j is
//   PV0(j-1) QK0(j) | PV1(j-1) QK1(j)
// so each softmax group works on tile j while the tensor core runs the other
// group's products (ping-pong).  Online softmax keeps a running row maximum m
// (log2 domain) and rescales O only when m grows by more than 8 (factor 256);
// the final O / l uses the same m, so the result is exact up to rounding.
//
// Work split (stream-K): unit = (batch, head, group of 256 query rows); its
// key tiles are the tiles any of its rows can see (fully masked tiles are never
// loaded).  All units' tiles are laid end to end and cut into one contiguous
// range per CTA.  A unit that one CTA covers entirely writes bf16 output
// directly; otherwise every piece writes fp32 partial (O, m, l) to the
// workspace and the last piece to finish (atomic counter) merges them.
#include "dz_internal.cuh"
#include "dz_ptx.cuh"

namespace dz {

namespace {

constexpr int NTHREADS = 384;
constexpr int WARP_TMA = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_ROPE = 2;   // warps 2..3
constexpr int WARP_SOFT = 4;   // warps 4..7 (group 0), 8..11 (group 1)
constexpr int ROPE_THREADS = (WARP_SOFT - WARP_ROPE) * 32;
constexpr int KV_STAGES = 2;
constexpr int TILE_BYTES = TILE_M * HEAD_DIM * 2;  // 32 KiB
constexpr int HALF_BYTES = TILE_BYTES / 2;         // 64 dims x 128 rows
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int SM_Q = 0;
constexpr int SM_K = SM_Q + Q_TILES * TILE_BYTES;
constexpr int SM_V = SM_K + KV_STAGES * TILE_BYTES;
constexpr int SM_BAR = SM_V + KV_STAGES * TILE_BYTES;
enum {
  B_Q_FULL = 0,
  B_Q_READY = 1,
  B_Q_EMPTY = 2,
  B_K_FULL = 3,
  B_K_READY = B_K_FULL + KV_STAGES,
  B_K_EMPTY = B_K_READY + KV_STAGES,
  B_V_FULL = B_K_EMPTY + KV_STAGES,
  B_V_EMPTY = B_V_FULL + KV_STAGES,
  B_S_FULL = B_V_EMPTY + KV_STAGES,
  B_P_FULL = B_S_FULL + Q_TILES,
  B_O_FULL = B_P_FULL + Q_TILES,
  B_O_FREE = B_O_FULL + Q_TILES,
  B_WG = B_O_FREE + Q_TILES,       // softmax-group rendezvous (split combine)
  B_DRAIN = B_WG + Q_TILES,
  B_COUNT = B_DRAIN + 1
};
constexpr int SM_MISC = SM_BAR + 256;         // tmem base, abort flag, combine flags
constexpr int SM_PREFIX = SM_MISC + 256;      // (MAX_Q_GROUPS + 1) ints
constexpr int SM_TOTAL = SM_PREFIX + (MAX_Q_GROUPS + 1) * 4;
constexpr int SMEM_BYTES = SM_TOTAL + 1024;   // alignment slack
static_assert(B_COUNT * 8 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct __align__(64) AttnParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_ck, tm_cv;
  __nv_bfloat16* out;
  float* ws;
  int* counters;
  int* status;
  RopeTables rope;
  ChunkGeom geom;
  SchedGeom sched;
  int B, H, n_qg;
  int rope_q, rope_k;
  long long W;
  int G;
  float scale_log2;
};

// One contiguous piece of a unit's key-tile list handled by this CTA.
struct Seg {
  int bh, qg;       // unit: batch*H + head, query group
  int t0, n;        // tile ordinals [t0, t0 + n) of the unit's list
  int e1, s2;       // the unit's list is [0, e1) then [s2, ...)
  bool full;        // this CTA covers the whole unit
  long long u0, u1; // flattened tile range of the unit
};

__device__ __forceinline__ bool seg_next(const AttnParams& p, const int* prefix, long long& pos,
                                         long long end, Seg& s) {
  if (pos >= end) return false;
  const int Tbh = prefix[p.n_qg];
  const long long bh = pos / Tbh;
  const int rem = static_cast<int>(pos - bh * Tbh);
  int lo = 0, hi = p.n_qg - 1;  // largest qg with prefix[qg] <= rem
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= rem) lo = mid; else hi = mid - 1;
  }
  const int Tq = prefix[lo + 1] - prefix[lo];
  s.bh = static_cast<int>(bh);
  s.qg = lo;
  s.t0 = rem - prefix[lo];
  long long seg_end = pos + (Tq - s.t0);
  if (seg_end > end) seg_end = end;
  s.n = static_cast<int>(seg_end - pos);
  s.full = (s.t0 == 0 && s.n == Tq);
  s.u0 = bh * Tbh + prefix[lo];
  s.u1 = s.u0 + Tq;
  int e1, s2, e2;
  unit_tiles(p.sched, lo, e1, s2, e2);
  s.e1 = e1;
  s.s2 = s2;
  pos = seg_end;
  return true;
}

__device__ __forceinline__ int seg_tile(const Seg& s, int i) {
  const int ord = s.t0 + i;
  return ord < s.e1 ? ord : s.s2 + (ord - s.e1);
}

struct KTile {
  bool cache;   // from the KV cache (DECODE) rather than the call's own k/v
  bool rope;    // rows need rotation (the call's own keys)
  int row0;     // first row in its source tensor
  int nvalid;   // rows < source length
  int vbase;    // key index of row0 in the call's key order (cache first)
};

__device__ __forceinline__ KTile ktile(const AttnParams& p, int kt) {
  KTile t;
  const SchedGeom& g = p.sched;
  if (g.mode == MODE_DECODE && kt < g.nkc) {
    t.cache = true;
    t.rope = false;
    t.row0 = kt * TILE_N;
    t.nvalid = min(TILE_N, g.cache_len - t.row0);
    t.vbase = t.row0;
  } else {
    const int st = (g.mode == MODE_DECODE) ? kt - g.nkc : kt;
    t.cache = false;
    t.rope = p.rope_k != 0;
    t.row0 = st * TILE_N;
    t.nvalid = min(TILE_N, g.Sk - t.row0);
    t.vbase = (g.mode == MODE_DECODE ? g.cache_len : 0) + t.row0;
  }
  return t;
}

// Visible keys of query token s (clamped to a real token), in the call's key
// order: [a0, a1) and [b0, b1).
__device__ __forceinline__ void row_ranges(const SchedGeom& g, int s, int& a0, int& a1, int& b0,
                                           int& b1) {
  a0 = 0;
  b0 = b1 = 0;
  if (g.mode == MODE_DECODE) {
    a1 = g.cache_len + g.L;
  } else if (g.mode == MODE_CROSS) {
    a1 = g.Sk;
  } else if (g.mode == MODE_PREFILL) {
    a1 = (s / g.L + 1) * g.L;
  } else {
    const int c = s / g.L;
    if (c < g.N) {
      a1 = (c + 1) * g.L;
    } else {
      const int i = c - g.N;
      a1 = i * g.L;
      b0 = (g.N + i) * g.L;
      b1 = b0 + g.L;
    }
  }
}

// Rotary position of token s of the call's q (or own k) tensor.
__device__ __forceinline__ void seq_pos(const AttnParams& p, int s, int& t, int& h, int& w) {
  int first = 0, ss = s;
  if (p.sched.mode == MODE_DECODE) {
    first = p.sched.N;
  } else if (p.sched.mode == MODE_TEACHER_FORCING && s >= p.sched.N * p.geom.L) {
    ss = s - p.sched.N * p.geom.L;
  }
  token_pos(p.geom, ss, first, t, h, w);
}

// Rotate row r of a 128x128 bf16 tile held as two 128B-swizzled halves.
__device__ __forceinline__ void rotate_tile_row(uint8_t* tile, int r, const RopeTables& rt, int t,
                                                int h, int w) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4* ptr = reinterpret_cast<uint4*>(tile + half * HALF_BYTES + r * 128 + ((c ^ (r & 7)) << 4));
      *ptr = rope_chunk(*ptr, rt, half * 32 + c * 4, t, h, w);
    }
  }
}

__device__ __forceinline__ long long cta_start(long long c, long long W, int G) {
  return c * W / G;
}
// The CTA whose range holds flattened tile x.
__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return static_cast<int>(((x + 1) * G - 1) / W);
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer() - t0 > DZ_WAIT_NS) return;
  }
}

}  // namespace

__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_attn_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + SM_Q;
  uint8_t* sK = smem + SM_K;
  uint8_t* sV = smem + SM_V;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + SM_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM_MISC + 4);
  volatile int* comb_flag = reinterpret_cast<volatile int*>(smem + SM_MISC + 8);  // [Q_TILES]
  int* prefix = reinterpret_cast<int*>(smem + SM_PREFIX);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- set-up: barriers, TMEM, per-group tile counts ----
  if (tid == 0) {
    mbar_init(&bar[B_Q_FULL], 1);
    mbar_init(&bar[B_Q_READY], ROPE_THREADS);
    mbar_init(&bar[B_Q_EMPTY], 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&bar[B_K_FULL + s], 1);
      mbar_init(&bar[B_K_READY + s], ROPE_THREADS);
      mbar_init(&bar[B_K_EMPTY + s], 1);
      mbar_init(&bar[B_V_FULL + s], 1);
      mbar_init(&bar[B_V_EMPTY + s], 1);
    }
    for (int q = 0; q < Q_TILES; ++q) {
      mbar_init(&bar[B_S_FULL + q], 1);
      mbar_init(&bar[B_P_FULL + q], 128);
      mbar_init(&bar[B_O_FULL + q], 1);
      mbar_init(&bar[B_O_FREE + q], 128);
      mbar_init(&bar[B_WG + q], 128);
    }
    mbar_init(&bar[B_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  for (int g = tid; g < p.n_qg; g += NTHREADS) prefix[g + 1] = unit_tile_count(p.sched, g);
  __syncthreads();
  if (warp == 0) {  // inclusive scan of the counts -> prefix[0..n_qg]
    int carry = 0;
    for (int base = 0; base < p.n_qg; base += 32) {
      const int g = base + lane;
      int v = (g < p.n_qg) ? prefix[g + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (g < p.n_qg) prefix[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) prefix[0] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long cstart = cta_start(blockIdx.x, p.W, p.G);
  const long long cend = cta_start(blockIdx.x + 1, p.W, p.G);

  if (warp == WARP_TMA) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      if (p.sched.nkc > 0) {
        tma_prefetch_desc(&p.tm_ck);
        tma_prefetch_desc(&p.tm_cv);
      }
      long long pos = cstart;
      Seg sg;
      int seg_i = 0;
      uint32_t k_iss = 0, v_iss = 0;  // K and V tiles issued so far
      int q_loads = 0;
      bool ok = true;
      while (ok && seg_next(p, prefix, pos, cend, sg)) {
        const int b = sg.bh / p.H, h = sg.bh - (sg.bh / p.H) * p.H;
        if (seg_i > 0 && !mbar_wait(&bar[B_Q_EMPTY], (seg_i - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(&bar[B_Q_FULL], Q_TILES * TILE_BYTES);
        for (int q = 0; q < Q_TILES; ++q) {
          const int row = sg.qg * Q_GROUP + q * TILE_M;
          tma_load_4d(sQ + q * TILE_BYTES, &p.tm_q, &bar[B_Q_FULL], 0, h, row, b);
          tma_load_4d(sQ + q * TILE_BYTES + HALF_BYTES, &p.tm_q, &bar[B_Q_FULL], 64, h, row, b);
        }
        ++q_loads;
        for (int i = 0; i < sg.n; ++i) {
          const int st = k_iss % KV_STAGES;
          const uint32_t ph = (k_iss / KV_STAGES) & 1;
          const KTile kt = ktile(p, seg_tile(sg, i));
          const CUtensorMap* mk = kt.cache ? &p.tm_ck : &p.tm_k;
          const CUtensorMap* mv = kt.cache ? &p.tm_cv : &p.tm_v;
          if (!mbar_wait(&bar[B_K_EMPTY + st], ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          mbar_expect_tx(&bar[B_K_FULL + st], TILE_BYTES);
          tma_load_4d(sK + st * TILE_BYTES, mk, &bar[B_K_FULL + st], 0, h, kt.row0, b);
          tma_load_4d(sK + st * TILE_BYTES + HALF_BYTES, mk, &bar[B_K_FULL + st], 64, h, kt.row0, b);
          ++k_iss;
          if (!mbar_wait(&bar[B_V_EMPTY + st], ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          mbar_expect_tx(&bar[B_V_FULL + st], TILE_BYTES);
          tma_load_4d(sV + st * TILE_BYTES, mv, &bar[B_V_FULL + st], 0, h, kt.row0, b);
          tma_load_4d(sV + st * TILE_BYTES + HALF_BYTES, mv, &bar[B_V_FULL + st], 64, h, kt.row0, b);
          ++v_iss;
        }
        ++seg_i;
      }
      // drain: every copy this thread issued has landed before the CTA exits
      // (on the normal path all of them were consumed and these return at once)
      if (q_loads > 0) drain_wait(&bar[B_Q_FULL], (q_loads - 1) & 1);
      for (uint32_t j = (k_iss > KV_STAGES ? k_iss - KV_STAGES : 0); j < k_iss; ++j)
        drain_wait(&bar[B_K_FULL + j % KV_STAGES], (j / KV_STAGES) & 1);
      for (uint32_t j = (v_iss > KV_STAGES ? v_iss - KV_STAGES : 0); j < v_iss; ++j)
        drain_wait(&bar[B_V_FULL + j % KV_STAGES], (j / KV_STAGES) & 1);
    }
  } else if (warp == WARP_MMA) {
    // ======================= tcgen05 issuer =======================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16(TILE_M, TILE_N, false);
      const uint32_t idesc_pv = idesc_bf16(TILE_M, HEAD_DIM, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      auto issue_qk = [&](int q, int st) {
        const uint32_t a0 = sQa + q * TILE_BYTES, b0 = sKa + st * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < HEAD_DIM / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          mma_ss(tmem + q * TILE_N, smem_desc(a0 + off, 16, 1024), smem_desc(b0 + off, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int q, int st, bool acc) {
        const uint32_t b0 = sVa + st * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < TILE_N / 16; ++kk) {
          mma_ts(tmem + 256 + q * HEAD_DIM, tmem + q * TILE_N + kk * 8,
                 smem_desc(b0 + kk * 16 * 128, HALF_BYTES, 1024), idesc_pv,
                 (acc || kk > 0) ? 1u : 0u);
        }
      };
      long long pos = cstart;
      Seg sg;
      int seg_i = 0;
      uint32_t it = 0, tn = 0;
      bool ok = true;
      while (ok && seg_next(p, prefix, pos, cend, sg)) {
        if (!mbar_wait(&bar[B_Q_READY], seg_i & 1, abort_flag, p.status)) break;
        tc_fence_after();
        int pst = 0;
        uint32_t pph = 0;
        for (int i = 0; i < sg.n; ++i, ++it, ++tn) {
          const int st = it % KV_STAGES;
          const uint32_t ph = (it / KV_STAGES) & 1;
          if (!mbar_wait(&bar[B_K_READY + st], ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          if (i == 0) {
            for (int q = 0; q < Q_TILES; ++q) {
              issue_qk(q, st);
              mma_commit(&bar[B_S_FULL + q]);
            }
          } else {
            if (!mbar_wait(&bar[B_V_FULL + pst], pph, abort_flag, p.status)) { ok = false; break; }
            for (int q = 0; q < Q_TILES; ++q) {
              if (i == 1 && seg_i > 0 &&
                  !mbar_wait(&bar[B_O_FREE + q], (seg_i - 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
              }
              if (!mbar_wait(&bar[B_P_FULL + q], (tn - 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_pv(q, pst, i > 1);
              if (q == Q_TILES - 1) mma_commit(&bar[B_V_EMPTY + pst]);
              issue_qk(q, st);
              mma_commit(&bar[B_S_FULL + q]);
            }
            if (!ok) break;
          }
          mma_commit(&bar[B_K_EMPTY + st]);
          pst = st;
          pph = ph;
        }
        if (!ok) break;
        // products of the segment's last tile
        if (!mbar_wait(&bar[B_V_FULL + pst], pph, abort_flag, p.status)) break;
        for (int q = 0; q < Q_TILES; ++q) {
          if (sg.n == 1 && seg_i > 0 &&
              !mbar_wait(&bar[B_O_FREE + q], (seg_i - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&bar[B_P_FULL + q], (tn - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(q, pst, sg.n > 1);
          mma_commit(&bar[B_O_FULL + q]);
        }
        if (!ok) break;
        mma_commit(&bar[B_V_EMPTY + pst]);
        mma_commit(&bar[B_Q_EMPTY]);
        ++seg_i;
      }
      // every issued MMA has completed before TMEM is released
      mma_commit(&bar[B_DRAIN]);
      drain_wait(&bar[B_DRAIN], 0);
    }
  } else if (warp < WARP_SOFT) {
    // ======================= rotary gate =======================
    const int r0 = tid - WARP_ROPE * 32;  // rows r0 and r0 + ROPE_THREADS of a tile
    long long pos = cstart;
    Seg sg;
    int seg_i = 0;
    uint32_t it = 0;
    bool ok = true;
    while (ok && seg_next(p, prefix, pos, cend, sg)) {
      if (!mbar_wait(&bar[B_Q_FULL], seg_i & 1, abort_flag, p.status)) break;
      if (p.rope_q) {
        for (int q = 0; q < Q_TILES; ++q) {
          for (int r = r0; r < TILE_M; r += ROPE_THREADS) {
            const int s = sg.qg * Q_GROUP + q * TILE_M + r;
            if (s < p.sched.Sq) {
              int t, h, w;
              seq_pos(p, s, t, h, w);
              rotate_tile_row(sQ + q * TILE_BYTES, r, p.rope, t, h, w);
            }
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_Q_READY]);
      for (int i = 0; i < sg.n; ++i, ++it) {
        const int st = it % KV_STAGES;
        const uint32_t ph = (it / KV_STAGES) & 1;
        if (!mbar_wait(&bar[B_K_FULL + st], ph, abort_flag, p.status)) { ok = false; break; }
        const KTile kt = ktile(p, seg_tile(sg, i));
        if (kt.rope) {
          for (int r = r0; r < kt.nvalid; r += ROPE_THREADS) {
            int t, h, w;
            seq_pos(p, kt.row0 + r, t, h, w);
            rotate_tile_row(sK + st * TILE_BYTES, r, p.rope, t, h, w);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bar[B_K_READY + st]);
      }
      ++seg_i;
    }
  } else {
    // ======================= softmax groups =======================
    const int q = (warp - WARP_SOFT) >> 2;           // Q tile of this group
    const int gtid = tid - (WARP_SOFT + 4 * q) * 32;  // 0..127 inside the group
    const int r = 32 * (warp & 3) + lane;            // TMEM lane = tile row
    const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_addr + q * TILE_N;
    const uint32_t tO = tmem + lane_addr + 256 + q * HEAD_DIM;
    const float sl2 = p.scale_log2;
    long long pos = cstart;
    Seg sg;
    int seg_i = 0;
    uint32_t tn = 0, wg_phase = 0;
    bool ok = true;
    while (ok && seg_next(p, prefix, pos, cend, sg)) {
      const int b = sg.bh / p.H, h = sg.bh - (sg.bh / p.H) * p.H;
      const int s_tok = sg.qg * Q_GROUP + q * TILE_M + r;
      const int s_eff = s_tok < p.sched.Sq ? s_tok : p.sched.Sq - 1;
      int a0, a1, b0, b1;
      row_ranges(p.sched, s_eff, a0, a1, b0, b1);
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < sg.n; ++i, ++tn) {
        if (!mbar_wait(&bar[B_S_FULL + q], tn & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const KTile kt = ktile(p, seg_tile(sg, i));
        const int la = max(0, min(TILE_N, a0 - kt.vbase));
        const int ha = max(0, min(kt.nvalid, a1 - kt.vbase));
        const int lb = max(0, min(TILE_N, b0 - kt.vbase));
        const int hb = max(0, min(kt.nvalid, b1 - kt.vbase));
        const bool full = (la == 0 && ha == TILE_N);
        uint32_t v[32];
        // pass 1: row maximum of the visible scores
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tS + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = c * 32 + j;
            float s = __uint_as_float(v[j]);
            if (!full && !((col >= la && col < ha) || (col >= lb && col < hb))) s = -INFINITY;
            mx = fmaxf(mx, s);
          }
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = m_new > m_run + RESCALE_THRESHOLD;
        const float alpha = need ? ex2(m_run - m_new) : 1.f;
        if (__any_sync(0xffffffffu, need) && i > 0) {
          // O holds tiles < i of this segment (its PV completed before S_FULL fired)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
            tmem_st32(tO + c * 32, v);
          }
          tmem_wait_st();
        }
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float mb = (m_run == -INFINITY) ? 0.f : m_run;
        // pass 2: probabilities, written as bf16 pairs over the first 64 columns of S
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tS + c * 32, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c * 32 + 2 * j;
            float s0 = __uint_as_float(v[2 * j]);
            float s1 = __uint_as_float(v[2 * j + 1]);
            if (!full) {
              if (!((col >= la && col < ha) || (col >= lb && col < hb))) s0 = -INFINITY;
              if (!((col + 1 >= la && col + 1 < ha) || (col + 1 >= lb && col + 1 < hb))) s1 = -INFINITY;
            }
            const float p0 = ex2(__fmaf_rn(s0, sl2, -mb));
            const float p1 = ex2(__fmaf_rn(s1, sl2, -mb));
            lsum += p0 + p1;
            pk[j] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        tmem_wait_st();
        l_run += lsum;
        tc_fence_before();
        mbar_arrive(&bar[B_P_FULL + q]);
      }
      if (!ok) break;
      // ---- epilogue of the segment ----
      if (!mbar_wait(&bar[B_O_FULL + q], seg_i & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const bool store_row = s_tok < p.sched.Sq;
      if (sg.full) {
        const float inv_l = 1.f / l_run;
        __nv_bfloat16* orow = p.out + ((static_cast<size_t>(b) * p.sched.Sq + (store_row ? s_tok : 0)) * p.H + h) * HEAD_DIM;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
          if (store_row) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * inv_l, __uint_as_float(v[2 * j + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&bar[B_O_FREE + q]);
      } else {
        // partial piece: fp32 (O, m, l) to this CTA's slot
        const bool first_piece = cta_start(blockIdx.x, p.W, p.G) >= sg.u0;
        const int slot = 2 * blockIdx.x + (first_piece ? 0 : 1);
        float* buf = p.ws + static_cast<size_t>(slot) * PART_FLOATS;
        float* orow = buf + static_cast<size_t>(q * TILE_M + r) * HEAD_DIM;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
        tc_fence_before();
        mbar_arrive(&bar[B_O_FREE + q]);
        float* ml = buf + static_cast<size_t>(Q_TILES) * TILE_M * HEAD_DIM + (q * TILE_M + r) * 2;
        ml[0] = m_run;
        ml[1] = l_run;
        __threadfence();
        mbar_arrive(&bar[B_WG + q]);
        if (!mbar_wait(&bar[B_WG + q], wg_phase & 1, abort_flag, p.status)) break;
        ++wg_phase;
        const int c_first = cta_of(sg.u0, p.W, p.G);
        const int c_last = cta_of(sg.u1 - 1, p.W, p.G);
        int* counter = p.counters + (static_cast<size_t>(sg.bh) * p.n_qg + sg.qg) * Q_TILES + q;
        if (gtid == 0) {
          const int old = atomicAdd(counter, 1);
          comb_flag[q] = (old == c_last - c_first) ? 1 : 0;
        }
        mbar_arrive(&bar[B_WG + q]);
        if (!mbar_wait(&bar[B_WG + q], wg_phase & 1, abort_flag, p.status)) break;
        ++wg_phase;
        if (comb_flag[q]) {
          __threadfence();
          float M = -INFINITY;
          for (int c2 = c_first; c2 <= c_last; ++c2) {
            const int sl = 2 * c2 + (cta_start(c2, p.W, p.G) >= sg.u0 ? 0 : 1);
            const float* ml2 = p.ws + static_cast<size_t>(sl) * PART_FLOATS +
                               static_cast<size_t>(Q_TILES) * TILE_M * HEAD_DIM + (q * TILE_M + r) * 2;
            M = fmaxf(M, __ldcg(ml2));
          }
          float Lsum = 0.f;
          for (int c2 = c_first; c2 <= c_last; ++c2) {
            const int sl = 2 * c2 + (cta_start(c2, p.W, p.G) >= sg.u0 ? 0 : 1);
            const float* ml2 = p.ws + static_cast<size_t>(sl) * PART_FLOATS +
                               static_cast<size_t>(Q_TILES) * TILE_M * HEAD_DIM + (q * TILE_M + r) * 2;
            const float m2 = __ldcg(ml2);
            if (m2 != -INFINITY) Lsum += __ldcg(ml2 + 1) * ex2(m2 - M);
          }
          const float inv_l = 1.f / Lsum;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float acc[32];
#pragma unroll
            for (int d = 0; d < 32; ++d) acc[d] = 0.f;
            for (int c2 = c_first; c2 <= c_last; ++c2) {
              const int sl = 2 * c2 + (cta_start(c2, p.W, p.G) >= sg.u0 ? 0 : 1);
              const float* b2 = p.ws + static_cast<size_t>(sl) * PART_FLOATS;
              const float m2 = __ldcg(b2 + static_cast<size_t>(Q_TILES) * TILE_M * HEAD_DIM + (q * TILE_M + r) * 2);
              if (m2 == -INFINITY) continue;
              const float wgt = ex2(m2 - M);
              const float4* o2 = reinterpret_cast<const float4*>(b2 + static_cast<size_t>(q * TILE_M + r) * HEAD_DIM + c * 32);
#pragma unroll
              for (int d = 0; d < 8; ++d) {
                const float4 x = __ldcg(o2 + d);
                acc[4 * d] += wgt * x.x;
                acc[4 * d + 1] += wgt * x.y;
                acc[4 * d + 2] += wgt * x.z;
                acc[4 * d + 3] += wgt * x.w;
              }
            }
            if (store_row) {
              __nv_bfloat16* orow2 = p.out + ((static_cast<size_t>(b) * p.sched.Sq + s_tok) * p.H + h) * HEAD_DIM + c * 32;
              uint4* dst = reinterpret_cast<uint4*>(orow2);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pack_bf16x2(acc[8 * j] * inv_l, acc[8 * j + 1] * inv_l),
                                    pack_bf16x2(acc[8 * j + 2] * inv_l, acc[8 * j + 3] * inv_l),
                                    pack_bf16x2(acc[8 * j + 4] * inv_l, acc[8 * j + 5] * inv_l),
                                    pack_bf16x2(acc[8 * j + 6] * inv_l, acc[8 * j + 7] * inv_l));
            }
          }
          if (gtid == 0) *counter = 0;  // ready for the next call
        }
      }
      ++seg_i;
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) {
    __syncwarp();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(chunk_attn_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  AttnParams p;
  p.tm_q = a.tm_q;
  p.tm_k = a.tm_k;
  p.tm_v = a.tm_v;
  p.tm_ck = a.tm_ck;
  p.tm_cv = a.tm_cv;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ws = a.ws;
  p.counters = a.counters;
  p.status = a.status;
  p.rope = a.rope;
  p.geom = a.geom;
  p.sched = a.sched;
  p.B = a.B;
  p.H = a.H;
  p.n_qg = a.n_qg;
  p.rope_q = a.rope_q;
  p.rope_k = a.rope_k;
  p.W = a.W;
  p.G = a.grid;
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HEAD_DIM));
  chunk_attn_kernel<<<a.grid, NTHREADS, SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dz
