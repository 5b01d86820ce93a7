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
//                 through a 2-stage ring (128B-swizzled, K-major rows of 128 dims);
//                 one commit after each tile's QK products frees its K stage and the
//                 previous tile's V stage (those PV products precede it in the queue).
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
// range per CTA (one CTA per unit when that is no slower).  Prefill and teacher
// forcing calls with many units first deal whole units round-robin in head-major
// order (a second instantiation of the kernel), so that the CTAs running together
// share a few heads' keys through L2, and split only the remaining units.  A unit that one
// CTA covers entirely writes bf16 output directly; otherwise each piece counts
// its arrival on the unit's counter, every piece but the last to arrive
// publishes fp32 partial (O, m, l) to the workspace, and the last one sums all
// pieces in CTA order (its own O read from TMEM in its place), so the result does
// not depend on the arrival order.  With the call's q and own k rotated once into a
// workspace beforehand (or given rotated), the rotary gate only passes tiles on.
//
// E4M3 variant (second template argument): q and k arrive rotated as E4M3 codes (one
// byte per element, one 128-byte swizzle row per token, 16 KiB per tile in the first
// half of each Q/K slot) and QK^T runs as kind::f8f6f4 products of K = 32; the
// multipliers of q and k are folded into the softmax scale.  V, P, O and the output
// are as in the bf16 kernel.
#include <type_traits>

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
constexpr int TILE_BYTES_E4M3 = TILE_M * HEAD_DIM;  // 16 KiB: 128 one-byte dims x 128 rows
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
// Registers per thread: the kernel is compiled for LAUNCH_REGS (3 warps per SM
// sub-partition); warpgroup 0 (producer, MMA, rotary) then gives registers to
// the two softmax warpgroups.  The split must add up to the launch budget.
constexpr int LAUNCH_REGS = 168;
constexpr int REGS_CTRL = 136;
constexpr int REGS_SOFT = 184;
static_assert(REGS_CTRL + 2 * REGS_SOFT == 3 * LAUNCH_REGS, "register split must match launch");

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr int SM_Q = 0;
constexpr int SM_K = SM_Q + Q_TILES * TILE_BYTES;
constexpr int SM_V = SM_K + KV_STAGES * TILE_BYTES;
constexpr int XPOSE_PITCH = 80;                        // bytes per row of a warp's transpose buffer
constexpr int XPOSE_WARP = 32 * XPOSE_PITCH;           // 32 rows x 64 data bytes (+16 pad)
constexpr int SM_X = SM_V + KV_STAGES * TILE_BYTES;    // 8 softmax warps' transpose buffers
constexpr int SM_BAR = SM_X + 8 * XPOSE_WARP;
enum {
  B_Q_FULL = 0,
  B_Q_READY = 1,
  B_Q_EMPTY = 2,
  B_K_FULL = 3,                     // K tile landed (tiles used as loaded)
  B_K_RAW = B_K_FULL + KV_STAGES,   // K tile landed (tiles the rotary gate must rotate)
  B_K_READY = B_K_RAW + KV_STAGES,  // rotated K tile released to the tensor core
  B_K_EMPTY = B_K_READY + KV_STAGES,  // tile's QK products done (and the previous tile's PV)
  B_V_FULL = B_K_EMPTY + KV_STAGES,
  B_S_FULL = B_V_FULL + KV_STAGES,
  B_P_FULL = B_S_FULL + Q_TILES,
  B_O_FULL = B_P_FULL + Q_TILES,
  B_O_FREE = B_O_FULL + Q_TILES,
  B_DRAIN = B_O_FREE + Q_TILES,
  B_COUNT = B_DRAIN + 1
};
constexpr int SM_MISC = SM_BAR + 256;         // tmem base, abort flag, combine flags
constexpr int SM_PREFIX = SM_MISC + 256;      // (MAX_Q_GROUPS + 1) ints
constexpr int SM_TB = SM_PREFIX + ((MAX_Q_GROUPS + 1) * 4 + 15) / 16 * 16;  // tail ranges (G + 1)
constexpr int SM_ROPE = SM_TB + ((MAX_GRID + 1) * 4 + 15) / 16 * 16;  // staged rotary rows
constexpr int SM_TOTAL = SM_ROPE + ROPE_STAGE_MAX * 8;
constexpr int SMEM_BYTES = SM_TOTAL + 1024;   // alignment slack
static_assert(B_COUNT * 8 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct __align__(64) AttnParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_ck, tm_cv;
  __nv_bfloat16* out;
  float* lse;  // null, or log2-domain softmax normaliser per (b, h, query row)
  float* ws;
  int* counters;
  int* status;
  long long out_elems;   // B * Sq * H * 128 (bounds-checked build)
  int ws_slots;          // partial-result slots of ws
  long long n_counters;  // split counters
  RopeTables rope;
  ChunkGeom geom;
  SchedGeom sched;
  int B, H, n_qg;
  int rope_q, rope_k;
  int stage_ok, stage_t0, stage_nt;
  unsigned W;  // total key tiles; W * G < 2^31 (checked on the host)
  int G;
  float scale_log2;
};

// Parameters of the schedule with whole-unit waves (prefill / teacher forcing):
// `waves` rounds of whole units dealt round-robin (CTA c takes unit c + k * G of the
// head-major order, so the CTAs that run together read the same few heads' keys
// and those come from L2), then CTA c takes flattened key tiles [tb[c], tb[c + 1])
// of the remaining units.
struct __align__(64) AttnParamsWaves : AttnParams {
  int waves;
  unsigned tb[MAX_GRID + 1];
};

// One contiguous piece of a unit's key-tile list handled by this CTA.
struct Seg {
  int bh, qg;       // unit: batch*H + head, query group
  int t0, n;        // tile ordinals [t0, t0 + n) of the unit's list
  int e1, s2;       // the unit's list is [0, e1) then [s2, ...)
  bool full;        // this CTA covers the whole unit
  unsigned u0, u1;  // flattened tile range of the unit
};

// Where a CTA is in its work list: whole units dealt so far (waves schedule), then
// its position in its range of flattened key tiles.
struct Cursor {
  int k;
  unsigned pos;
};

// The CTA's next segment: with the waves schedule first its whole units, then (both
// schedules) the pieces of its contiguous range of flattened key tiles.
template <class P>
__device__ __forceinline__ bool seg_next(const P& p, const int* prefix, Cursor& cur,
                                         unsigned end, Seg& s) {
  const int Tbh = prefix[p.n_qg];
  if constexpr (std::is_same<P, AttnParamsWaves>::value) {
    if (cur.k < p.waves) {
      const int u = static_cast<int>(blockIdx.x) + cur.k * p.G;
      ++cur.k;
      const int bh = u / p.n_qg, qg = u - (u / p.n_qg) * p.n_qg;
      const int Tq = prefix[qg + 1] - prefix[qg];
      s.bh = bh;
      s.qg = qg;
      s.t0 = 0;
      s.n = Tq;
      s.full = true;
      s.u0 = static_cast<unsigned>(bh) * Tbh + prefix[qg];
      s.u1 = s.u0 + Tq;
      int e1, s2, e2;
      unit_tiles(p.sched, qg, e1, s2, e2);
      s.e1 = e1;
      s.s2 = s2;
      return true;
    }
  }
  unsigned& pos = cur.pos;
  if (pos >= end) return false;
  const unsigned bh = pos / static_cast<unsigned>(Tbh);
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
  unsigned seg_end = pos + static_cast<unsigned>(Tq - s.t0);
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

// Rotate row r of a 128x128 bf16 tile held as two 128B-swizzled halves (16-byte
// chunk c of row r sits at half (c / 8), slot (c % 8) ^ (r % 8)).  The table
// values of four chunks are loaded before their shared-memory read-modify-write
// so that the loads overlap.  `rt.tab` may point to shared or global memory.
__device__ __forceinline__ void rotate_tile_row(uint8_t* tile, int r, const RopeTables& rt, int t,
                                                int h, int w, int* status) {
  uint8_t* row = tile + r * 128;
#pragma unroll
  for (int b4 = 0; b4 < 4; ++b4) {
    float2 cs[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        cs[4 * k + i] = rt.tab[rope_index_checked(rt, (b4 * 4 + k) * 4 + i, t, h, w, status)];
    }
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = b4 * 4 + k;
      v[k] = *reinterpret_cast<const uint4*>(row + (c >> 3) * HALF_BYTES + (((c & 7) ^ (r & 7)) << 4));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k].x = rope_pair(v[k].x, cs[4 * k + 0]);
      v[k].y = rope_pair(v[k].y, cs[4 * k + 1]);
      v[k].z = rope_pair(v[k].z, cs[4 * k + 2]);
      v[k].w = rope_pair(v[k].w, cs[4 * k + 3]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = b4 * 4 + k;
      *reinterpret_cast<uint4*>(row + (c >> 3) * HALF_BYTES + (((c & 7) ^ (r & 7)) << 4)) = v[k];
    }
  }
}


// Scores of columns outside [la, ha) and [lb, hb) become -inf (32 columns from col0).
__device__ __forceinline__ void mask_cols(uint32_t (&v)[32], int col0, int la, int ha, int lb,
                                          int hb) {
  const uint32_t keep = range_bits(la - col0, ha - col0) | range_bits(lb - col0, hb - col0);
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = ((keep >> j) & 1u) ? v[j] : 0xff800000u;  // -inf
}

__device__ __forceinline__ float max32(const uint32_t (&v)[32]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = __uint_as_float(v[k]);
#pragma unroll
  for (int j = 8; j < 32; ++j) m[j & 7] = fmaxf(m[j & 7], __uint_as_float(v[j]));
  return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// p = 2^(s * scale_log2 - mb) for 32 scores, packed as 16 bf16 pairs into pk[off, off + 16);
// returns the fp32 sum of the 32 probabilities.  Pairs go through packed
// two-lane fp32 FMA/add instructions.
__device__ __forceinline__ float exp_pack(const uint32_t (&v)[32], uint32_t (&pk)[32], int off,
                                          float sl2, float mb) {
  const float2 sc = make_float2(sl2, sl2), nm = make_float2(-mb, -mb);
  float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 x = ffma2(make_float2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])), sc, nm);
    const float2 pp = make_float2(ex2(x.x), ex2(x.y));
    s2[j & 1] = fadd2(s2[j & 1], pp);
    pk[off + j] = pack_bf16x2(pp.x, pp.y);
  }
  const float2 t = fadd2(s2[0], s2[1]);
  return t.x + t.y;
}

// Rotate row r of a swizzled 128x128 bf16 tile (shared address `tile`) when the
// pair split (PT, PH, PW) is known at compile time and the row's t-, h- and
// w-table rows sit in shared memory at addresses tt, th, tw: every table read is
// one shared load at a constant offset.
template <int PT, int PH, int PW>
__device__ __forceinline__ void rotate_tile_row_split(uint32_t tile, int r, uint32_t tt,
                                                      uint32_t th, uint32_t tw) {
  static_assert(PT + PH + PW == HEAD_DIM / 2, "pair split");
  const uint32_t row = tile + r * 128;
#pragma unroll
  for (int b4 = 0; b4 < 4; ++b4) {
    float2 cs[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int j = b4 * 16 + k;
      cs[k] = lds_f2(j < PT ? tt + 8 * j : (j < PT + PH ? th + 8 * (j - PT) : tw + 8 * (j - PT - PH)));
    }
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = b4 * 4 + k;
      v[k] = lds_u4(row + (c >> 3) * HALF_BYTES + (((c & 7) ^ (r & 7)) << 4));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[k].x = rope_pair(v[k].x, cs[4 * k + 0]);
      v[k].y = rope_pair(v[k].y, cs[4 * k + 1]);
      v[k].z = rope_pair(v[k].z, cs[4 * k + 2]);
      v[k].w = rope_pair(v[k].w, cs[4 * k + 3]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = b4 * 4 + k;
      sts_u4(row + (c >> 3) * HALF_BYTES + (((c & 7) ^ (r & 7)) << 4), v[k]);
    }
  }
}

__device__ __forceinline__ unsigned cta_start(unsigned c, unsigned W, int G) {
  return c * W / static_cast<unsigned>(G);
}
// The CTA whose range holds flattened tile x.
__device__ __forceinline__ int cta_of(unsigned x, unsigned W, int G) {
  return static_cast<int>(((x + 1) * static_cast<unsigned>(G) - 1) / W);
}
// The same with explicit ranges (staged in shared memory): the largest c with tb[c] <= x.
__device__ __forceinline__ int cta_of(const unsigned* tb, int G, unsigned x) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tb[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}


}  // namespace

template <class P, bool F8>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_attn_kernel(const __grid_constant__ P p) {
  constexpr bool kWaves = std::is_same<P, AttnParamsWaves>::value;
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
  unsigned* tb = reinterpret_cast<unsigned*>(smem + SM_TB);

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
      mbar_init(&bar[B_K_RAW + s], 1);
      mbar_init(&bar[B_K_READY + s], ROPE_THREADS);
      mbar_init(&bar[B_K_EMPTY + s], 1);
      mbar_init(&bar[B_V_FULL + s], 1);
    }
    for (int q = 0; q < Q_TILES; ++q) {
      mbar_init(&bar[B_S_FULL + q], 1);
      mbar_init(&bar[B_P_FULL + q], 128);
      mbar_init(&bar[B_O_FULL + q], 1);
      mbar_init(&bar[B_O_FREE + q], 128);
    }
    mbar_init(&bar[B_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (p.sched.nkc > 0) {
      tma_prefetch_desc(&p.tm_ck);
      tma_prefetch_desc(&p.tm_cv);
    }
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  for (int g = tid; g < p.n_qg; g += NTHREADS) prefix[g + 1] = unit_tile_count(p.sched, g);
  if constexpr (kWaves) {
    for (int c = tid; c <= p.G; c += NTHREADS) tb[c] = p.tb[c];
  }
  // rotary view: the call's table rows copied to shared memory when they fit
  RopeTables rope = p.rope;
  if (p.stage_ok) {
    float2* st_tab = reinterpret_cast<float2*>(smem + SM_ROPE);
    const int nt = p.stage_nt * p.rope.pt, nh = p.geom.gh * p.rope.ph, nw = p.geom.gw * p.rope.pw;
    const float2* gt = p.rope.tab + p.rope.off_t + p.stage_t0 * p.rope.pt;
    const float2* gh = p.rope.tab + p.rope.off_h;
    const float2* gw = p.rope.tab + p.rope.off_w;
    for (int i = tid; i < nt + nh + nw; i += NTHREADS) {
      const long long gi = i < nt ? p.rope.off_t + static_cast<long long>(p.stage_t0) * p.rope.pt + i
                                  : (i < nt + nh ? p.rope.off_h + i - nt : p.rope.off_w + i - nt - nh);
      if (in_bounds(gi, p.rope.n, p.status))
        st_tab[i] = i < nt ? gt[i] : (i < nt + nh ? gh[i - nt] : gw[i - nt - nh]);
    }
    rope.tab = st_tab;
    rope.off_t = -p.stage_t0 * p.rope.pt;
    rope.off_h = nt;
    rope.off_w = nt + nh;
    rope.n = nt + nh + nw;
  }
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

  Cursor cstart;
  unsigned cend;
  if constexpr (kWaves) {
    cstart = {0, p.tb[blockIdx.x]};
    cend = p.tb[blockIdx.x + 1];
  } else {
    cstart = {0, cta_start(blockIdx.x, p.W, p.G)};
    cend = cta_start(blockIdx.x + 1, p.W, p.G);
  }

  if (warp < WARP_SOFT) {
  regs_dec<REGS_CTRL>();
  if (warp == WARP_TMA) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      Cursor pos = cstart;
      Seg sg;
      int seg_i = 0;
      uint32_t k_iss = 0, v_iss = 0;  // K and V tiles issued so far
      // loads issued per stage on K_FULL (used as loaded) and K_RAW (to be rotated);
      // each of those barriers has exactly one consumer that takes its phases in order
      uint32_t kf_cnt[KV_STAGES] = {0, 0}, kr_cnt[KV_STAGES] = {0, 0};
      int q_loads = 0;
      bool ok = true;
      while (ok && seg_next(p, prefix, pos, cend, sg)) {
        const int b = sg.bh / p.H, h = sg.bh - (sg.bh / p.H) * p.H;
        // Q of this segment: the previous segment's last QK products must be done
        if (seg_i > 0 && !mbar_wait(&bar[B_Q_EMPTY], (seg_i - 1) & 1, abort_flag, p.status)) break;
        mbar_expect_tx(&bar[B_Q_FULL], Q_TILES * (F8 ? TILE_BYTES_E4M3 : TILE_BYTES));
        for (int q = 0; q < Q_TILES; ++q) {
          const int row = sg.qg * Q_GROUP + q * TILE_M;
          tma_load_4d(sQ + q * TILE_BYTES, &p.tm_q, &bar[B_Q_FULL], 0, h, row, b);
          if constexpr (!F8)
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
          uint64_t* kb = &bar[(kt.rope ? B_K_RAW : B_K_FULL) + st];
          mbar_expect_tx(kb, F8 ? TILE_BYTES_E4M3 : TILE_BYTES);
          tma_load_4d(sK + st * TILE_BYTES, mk, kb, 0, h, kt.row0, b);
          if constexpr (!F8) tma_load_4d(sK + st * TILE_BYTES + HALF_BYTES, mk, kb, 64, h, kt.row0, b);
          if (kt.rope) ++kr_cnt[st]; else ++kf_cnt[st];
          ++k_iss;
          // the V stage held V(t - 2), whose products were issued before QK(t - 1): the
          // single commit after tile t - 1's QK products covers them
          if (v_iss >= 2) {
            const uint32_t tp = v_iss - 1;
            if (!mbar_wait(&bar[B_K_EMPTY + tp % KV_STAGES], (tp / KV_STAGES) & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
          }
          mbar_expect_tx(&bar[B_V_FULL + st], TILE_BYTES);
          tma_load_4d(sV + st * TILE_BYTES, mv, &bar[B_V_FULL + st], 0, h, kt.row0, b);
          tma_load_4d(sV + st * TILE_BYTES + HALF_BYTES, mv, &bar[B_V_FULL + st], 64, h, kt.row0, b);
          ++v_iss;
        }
        ++seg_i;
      }
      // drain: every copy this thread issued has landed before the CTA exits
      // (on the normal path all of them were consumed and these return at once)
      if (q_loads > 0) mbar_drain(&bar[B_Q_FULL], (q_loads - 1) & 1);
      for (int st = 0; st < KV_STAGES; ++st) {
        if (kf_cnt[st] > 0) mbar_drain(&bar[B_K_FULL + st], (kf_cnt[st] - 1) & 1);
        if (kr_cnt[st] > 0) mbar_drain(&bar[B_K_RAW + st], (kr_cnt[st] - 1) & 1);
      }
      for (uint32_t j = (v_iss > KV_STAGES ? v_iss - KV_STAGES : 0); j < v_iss; ++j)
        mbar_drain(&bar[B_V_FULL + j % KV_STAGES], (j / KV_STAGES) & 1);
    }
  } else if (warp == WARP_MMA) {
    // ======================= tcgen05 issuer =======================
    if (lane == 0) {
      const uint32_t idesc_qk = F8 ? idesc_e4m3(TILE_M, TILE_N) : idesc_bf16(TILE_M, TILE_N, false);
      const uint32_t idesc_pv = idesc_bf16(TILE_M, HEAD_DIM, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      // descriptors: only the low word (start address) changes between the K-steps
      const uint32_t q_lo = desc_lo(sQa, 16), k_lo = desc_lo(sKa, 16), v_lo = desc_lo(sVa, HALF_BYTES);
      auto issue_qk = [&](int q, int st) {
        const uint32_t a0 = q_lo + ((q * TILE_BYTES) >> 4), b0 = k_lo + ((st * TILE_BYTES) >> 4);
        const uint32_t d = tmem + q * TILE_N;
        if constexpr (F8) {
          // one 128-byte row per token: the four K = 32 steps walk along it
#pragma unroll
          for (int kk = 0; kk < HEAD_DIM / 32; ++kk) {
            const uint32_t off = (kk * 32) >> 4;
            mma_ss_e4m3(d, desc_join(a0 + off), desc_join(b0 + off), idesc_qk, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < HEAD_DIM / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
            mma_ss(d, desc_join(a0 + off), desc_join(b0 + off), idesc_qk, kk > 0 ? 1u : 0u);
          }
        }
      };
      auto issue_pv = [&](int q, int st, bool acc) {
        const uint32_t b0 = v_lo + ((st * TILE_BYTES) >> 4);
        const uint32_t d = tmem + 256 + q * HEAD_DIM, a = tmem + q * TILE_N;
#pragma unroll
        for (int kk = 0; kk < TILE_N / 16; ++kk) {
          mma_ts(d, a + kk * 8, desc_join(b0 + ((kk * 16 * 128) >> 4)), idesc_pv,
                 (acc || kk > 0) ? 1u : 0u);
        }
      };
      Cursor pos = cstart;
      Seg sg;
      int seg_i = 0;
      uint32_t it = 0, tn = 0;
      uint32_t kr_par = 0;  // bit s: parity of the next K_READY phase on stage s
      uint32_t kf_par = 0;  // bit s: parity of the next K_FULL phase on stage s
      bool ok = true;
      while (ok && seg_next(p, prefix, pos, cend, sg)) {
        if (!mbar_wait(&bar[B_Q_READY], seg_i & 1, abort_flag, p.status)) break;
        tc_fence_after();
        int pst = 0;
        uint32_t pph = 0;
        for (int i = 0; i < sg.n; ++i, ++it, ++tn) {
          const int st = it % KV_STAGES;
          const uint32_t ph = (it / KV_STAGES) & 1;
          const bool rot = ktile(p, seg_tile(sg, i)).rope;
          bool got;
          if (rot) {
            got = mbar_wait(&bar[B_K_READY + st], (kr_par >> st) & 1, abort_flag, p.status);
            kr_par ^= 1u << st;
          } else {
            got = mbar_wait(&bar[B_K_FULL + st], (kf_par >> st) & 1, abort_flag, p.status);
            kf_par ^= 1u << st;
          }
          if (!got) { ok = false; break; }
          tc_fence_after();
          const bool last = (i == sg.n - 1);
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
              issue_qk(q, st);
              mma_commit(&bar[B_S_FULL + q]);
            }
            if (!ok) break;
          }
          mma_commit(&bar[B_K_EMPTY + st]);
          if (last) mma_commit(&bar[B_Q_EMPTY]);  // Q may be replaced once these QK are done
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
        ++seg_i;
      }
      // every issued MMA has completed before TMEM is released
      mma_commit(&bar[B_DRAIN]);
      mbar_drain(&bar[B_DRAIN], 0);
    }
  } else {
    // ======================= rotary gate =======================
    const int r0 = tid - WARP_ROPE * 32;  // rows r0 + k * ROPE_THREADS of a tile
    // fast path: tables staged in shared memory and the 22/21/21 split
    const bool fast = p.stage_ok && p.rope.pt == 22 && p.rope.ph == 21 && p.rope.pw == 21;
    const uint32_t st_base = smem_u32(smem + SM_ROPE);
    const uint32_t st_h = st_base + 8 * (p.stage_nt * 22);
    const uint32_t st_w = st_h + 8 * (p.geom.gh * 21);
    auto rotate_row = [&](uint8_t* tile, int r, int t, int h, int w) {
      if (fast) {
        rotate_tile_row_split<22, 21, 21>(smem_u32(tile), r, st_base + 8 * ((t - p.stage_t0) * 22),
                                          st_h + 8 * (h * 21), st_w + 8 * (w * 21));
      } else {
        rotate_tile_row(tile, r, rope, t, h, w, p.status);
      }
    };
    Cursor pos = cstart;
    Seg sg;
    int seg_i = 0;
    uint32_t it = 0;
    uint32_t raw_par = 0;  // bit s: parity of the next K_RAW phase on stage s
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
              rotate_row(sQ + q * TILE_BYTES, r, t, h, w);
            }
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_Q_READY]);
      for (int i = 0; i < sg.n; ++i, ++it) {
        const KTile kt = ktile(p, seg_tile(sg, i));
        if (!kt.rope) continue;  // cache tiles go to the tensor core as loaded
        const int st = it % KV_STAGES;
        if (!mbar_wait(&bar[B_K_RAW + st], (raw_par >> st) & 1, abort_flag, p.status)) { ok = false; break; }
        raw_par ^= 1u << st;
        for (int r = r0; r < kt.nvalid; r += ROPE_THREADS) {
          int t, h, w;
          seq_pos(p, kt.row0 + r, t, h, w);
          rotate_row(sK + st * TILE_BYTES, r, t, h, w);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bar[B_K_READY + st]);
      }
      ++seg_i;
    }
  }
  } else {
    regs_inc<REGS_SOFT>();
    // ======================= softmax groups =======================
    const int q = (warp - WARP_SOFT) >> 2;           // Q tile of this group
    const int gtid = tid - (WARP_SOFT + 4 * q) * 32;  // 0..127 inside the group
    const int quarter = warp & 3;                    // TMEM lane quarter of this warp
    const int r = 32 * quarter + lane;               // TMEM lane = tile row
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quarter) << 16;
    const uint32_t tS = tmem + lane_addr + q * TILE_N;
    const uint32_t tO = tmem + lane_addr + 256 + q * HEAD_DIM;
    uint8_t* xp = smem + SM_X + (warp - WARP_SOFT) * XPOSE_WARP;  // this warp's transpose buffer
    const float sl2 = p.scale_log2;
    Cursor pos = cstart;
    Seg sg;
    int seg_i = 0;
    uint32_t tn = 0;
    bool ok = true;
    while (ok && seg_next(p, prefix, pos, cend, sg)) {
      const int b = sg.bh / p.H, h = sg.bh - (sg.bh / p.H) * p.H;
      const int row0 = sg.qg * Q_GROUP + q * TILE_M + 32 * quarter;  // token of this warp's lane 0
      const int s_tok = row0 + lane;
      const int s_eff = s_tok < p.sched.Sq ? s_tok : p.sched.Sq - 1;
      int a0, a1, b0, b1;
      row_ranges(p.sched, s_eff, a0, a1, b0, b1);
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < sg.n; ++i, ++tn) {
        // the tile's visible-column ranges, worked out before its scores are ready
        const KTile kt = ktile(p, seg_tile(sg, i));
        const int la = max(0, min(TILE_N, a0 - kt.vbase));
        const int ha = max(0, min(kt.nvalid, a1 - kt.vbase));
        const int lb = max(0, min(TILE_N, b0 - kt.vbase));
        const int hb = max(0, min(kt.nvalid, b1 - kt.vbase));
        const bool full = (la == 0 && ha == TILE_N);
        if (!mbar_wait(&bar[B_S_FULL + q], tn & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t v0[32], v1[32], v2[32], v3[32];
        tmem_ld32(tS, v0);
        tmem_ld32(tS + 32, v1);
        tmem_ld32(tS + 64, v2);
        tmem_ld32(tS + 96, v3);
        tmem_wait_ld();
        if (!full) {
          mask_cols(v0, 0, la, ha, lb, hb);
          mask_cols(v1, 32, la, ha, lb, hb);
          mask_cols(v2, 64, la, ha, lb, hb);
          mask_cols(v3, 96, la, ha, lb, hb);
        }
        const float mx = fmaxf(fmaxf(max32(v0), max32(v1)), fmaxf(max32(v2), max32(v3)));
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = m_new > m_run + RESCALE_THRESHOLD;
        const float alpha = need ? ex2(m_run - m_new) : 1.f;
        if (__any_sync(0xffffffffu, need) && i > 0) {
          // O holds tiles < i of this segment (its PV completed before S_FULL fired)
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t v[16];
            tmem_ld16(tO + c * 16, v);
            tmem_wait_ld();
            uint32_t w16[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w16[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
            tmem_st16(tO + c * 16, w16);
          }
          tmem_wait_st();
        }
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float mb = (m_run == -INFINITY) ? 0.f : m_run;
        // probabilities, written as bf16 pairs over the first 64 columns of S
        uint32_t pk0[32], pk1[32];
        const float lsum = exp_pack(v0, pk0, 0, sl2, mb) + exp_pack(v1, pk0, 16, sl2, mb) +
                           exp_pack(v2, pk1, 0, sl2, mb) + exp_pack(v3, pk1, 16, sl2, mb);
        tmem_st32(tS, pk0);
        tmem_st32(tS + 32, pk1);
        tmem_wait_st();
        l_run += lsum;
        tc_fence_before();
        mbar_arrive(&bar[B_P_FULL + q]);
      }
      if (!ok) break;
      // ---- epilogue of the segment ----
      if (!mbar_wait(&bar[B_O_FULL + q], seg_i & 1, abort_flag, p.status)) break;
      tc_fence_after();
      if (sg.full) {
        // bf16 out = O / l; each 32-column chunk goes through the warp's transpose
        // buffer so that global stores cover 64 contiguous bytes of 8 rows at a time
        const float inv_l = 1.f / l_run;
        if (p.lse && s_tok < p.sched.Sq) {
          const long long li = (static_cast<long long>(b) * p.H + h) * p.sched.Sq + s_tok;
          if (in_bounds(li, p.out_elems / HEAD_DIM, p.status)) p.lse[li] = m_run + __log2f(l_run);
        }
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before();
            mbar_arrive(&bar[B_O_FREE + q]);
          }
          uint4* xrow = reinterpret_cast<uint4*>(xp + lane * XPOSE_PITCH);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            xrow[j] = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * j]) * inv_l, __uint_as_float(v[8 * j + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * j + 2]) * inv_l, __uint_as_float(v[8 * j + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * j + 4]) * inv_l, __uint_as_float(v[8 * j + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * j + 6]) * inv_l, __uint_as_float(v[8 * j + 7]) * inv_l));
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int task = lane + 32 * k;
            const int rr = task >> 2, piece = task & 3;
            const int s = row0 + rr;
            const uint4 val = *reinterpret_cast<const uint4*>(xp + rr * XPOSE_PITCH + piece * 16);
            const long long oi = ((static_cast<long long>(b) * p.sched.Sq + s) * p.H + h) * HEAD_DIM + c * 32 + piece * 8;
            if (s < p.sched.Sq && in_bounds(oi + 7, p.out_elems, p.status))
              *reinterpret_cast<uint4*>(p.out + oi) = val;
          }
          __syncwarp();
        }
      } else {
        // partial piece of a unit split across CTAs.  Its (bh, qg, q) counter
        // counts arrivals in the low 16 bits and published partials in the high
        // bits.  Every piece but the last to arrive publishes fp32 (O, m, l) in
        // its slot; the last one waits for those and merges them with its own O,
        // still in TMEM.  Slot layout: O as [32 column quads][Q_TILES * TILE_M
        // rows] float4 (one warp access = 512 contiguous bytes), then (m, l) per
        // row as float2.
        constexpr int ROWS = Q_TILES * TILE_M;
        const int row_l = q * TILE_M + r;
        const int c_first = kWaves ? cta_of(tb, p.G, sg.u0) : cta_of(sg.u0, p.W, p.G);
        const int c_last = kWaves ? cta_of(tb, p.G, sg.u1 - 1) : cta_of(sg.u1 - 1, p.W, p.G);
        const int np = c_last - c_first + 1;
        // slot of the piece held by CTA c: its first segment (slot 2c) unless the
        // unit began before c's range, which only the first piece's CTA can see
        const unsigned start_first = kWaves ? tb[c_first] : cta_start(c_first, p.W, p.G);
        const int slot0 = 2 * c_first + (start_first == sg.u0 ? 0 : 1);
        const int me = static_cast<int>(blockIdx.x) - c_first;  // piece index
        auto slot_of = [&](int k) {
          const int sl = k == 0 ? slot0 : 2 * (c_first + k);
          return in_bounds(sl, p.ws_slots, p.status) ? sl : 0;
        };
        long long ci = (static_cast<long long>(sg.bh) * p.n_qg + sg.qg) * Q_TILES + q;
        if (!in_bounds(ci, p.n_counters, p.status)) ci = 0;
        int* counter = p.counters + ci;
        if (gtid == 0) {
          const int old = atomicAdd(counter, 1);
          comb_flag[q] = ((old & 0xffff) == np - 1) ? 1 : 0;
        }
        named_bar_sync(1 + q, 128);
        // (both paths below pass another group barrier before comb_flag[q] can be rewritten)
        const bool last = comb_flag[q] != 0;
        if (!last) {
          float4* o4 = reinterpret_cast<float4*>(p.ws + static_cast<size_t>(slot_of(me)) * PART_FLOATS);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
            if (c == 3) {
              tc_fence_before();
              mbar_arrive(&bar[B_O_FREE + q]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
              o4[(c * 8 + j) * ROWS + row_l] =
                  make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                              __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
          reinterpret_cast<float2*>(p.ws + static_cast<size_t>(slot_of(me)) * PART_FLOATS +
                                    static_cast<size_t>(ROWS) * HEAD_DIM)[row_l] =
              make_float2(m_run, l_run);
          __threadfence();
          named_bar_sync(1 + q, 128);
          if (gtid == 0) atomicAdd(counter, 1 << 16);
        } else {
          // wait until the other np - 1 pieces have published
          if (gtid == 0) {
            const int want = (np - 1) << 16;
            const uint64_t t0 = globaltimer();
            uint32_t n = 0;
            while ((ld_acquire_gpu(counter) & ~0xffff) != want) {
              if (((++n) & 63u) == 0u) {
                if (*abort_flag) break;
                if (globaltimer() - t0 > DZ_WAIT_NS) {
                  *abort_flag = 1;
                  atomicOr(p.status, DZ_DEV_TIMEOUT);
                  break;
                }
              }
            }
          }
          named_bar_sync(1 + q, 128);
          if (*abort_flag) {
            ok = false;
            break;
          }
          __threadfence();
          // Every piece's weight and sum in CTA order, with this piece's own (m, l) in
          // its place, then the output 32 columns at a time as the sum over the pieces
          // in that order: the result does not depend on which piece arrived last.  A
          // row without visible keys in a piece adds nothing.
          auto ml_of = [&](int k) -> float2 {
            if (k == me) return make_float2(m_run, l_run);
            return __ldcg(reinterpret_cast<const float2*>(
                       p.ws + static_cast<size_t>(slot_of(k)) * PART_FLOATS +
                       static_cast<size_t>(ROWS) * HEAD_DIM) + row_l);
          };
          float M = -INFINITY;
          for (int k = 0; k < np; ++k) M = fmaxf(M, ml_of(k).x);
          float Lsum = 0.f;
          for (int k = 0; k < np; ++k) {
            const float2 mk = ml_of(k);
            Lsum += (mk.x == -INFINITY) ? 0.f : mk.y * ex2(mk.x - M);
          }
          const float invL = 1.f / Lsum;
          if (p.lse && s_tok < p.sched.Sq) {
            const long long li = (static_cast<long long>(b) * p.H + h) * p.sched.Sq + s_tok;
            if (in_bounds(li, p.out_elems / HEAD_DIM, p.status)) p.lse[li] = M + __log2f(Lsum);
          }
          // the first other piece's next 32 columns are loaded while this pass runs
          const int kp = me == 0 ? 1 : 0;
          const float4* srcp = reinterpret_cast<const float4*>(p.ws + static_cast<size_t>(slot_of(kp)) * PART_FLOATS);
          float4 nxt[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) nxt[j] = __ldcg(srcp + j * ROWS + row_l);
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {  // 32 output columns per pass
            float4 cur[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
            if (g < 3) {
#pragma unroll
              for (int j = 0; j < 8; ++j) nxt[j] = __ldcg(srcp + ((g + 1) * 8 + j) * ROWS + row_l);
            }
            float acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0.f;
            for (int k = 0; k < np; ++k) {
              const float mk = ml_of(k).x;
              const float sk = (mk == -INFINITY) ? 0.f : ex2(mk - M);
              if (k == me) {
                uint32_t v[32];
                tmem_ld32(tO + g * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[j] += __uint_as_float(v[j]) * sk;
              } else if (k == kp) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  acc[4 * j] += cur[j].x * sk;
                  acc[4 * j + 1] += cur[j].y * sk;
                  acc[4 * j + 2] += cur[j].z * sk;
                  acc[4 * j + 3] += cur[j].w * sk;
                }
              } else {
                const float4* src = reinterpret_cast<const float4*>(
                    p.ws + static_cast<size_t>(slot_of(k)) * PART_FLOATS);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 o = __ldcg(src + (g * 8 + j) * ROWS + row_l);
                  acc[4 * j] += o.x * sk;
                  acc[4 * j + 1] += o.y * sk;
                  acc[4 * j + 2] += o.z * sk;
                  acc[4 * j + 3] += o.w * sk;
                }
              }
            }
            if (g == 3) {
              tc_fence_before();
              mbar_arrive(&bar[B_O_FREE + q]);
            }
            // bf16 row chunk through the warp's transpose buffer, then 64-byte row pieces
            uint4* xrow = reinterpret_cast<uint4*>(xp + lane * XPOSE_PITCH);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              xrow[j] = make_uint4(pack_bf16x2(acc[8 * j] * invL, acc[8 * j + 1] * invL),
                                   pack_bf16x2(acc[8 * j + 2] * invL, acc[8 * j + 3] * invL),
                                   pack_bf16x2(acc[8 * j + 4] * invL, acc[8 * j + 5] * invL),
                                   pack_bf16x2(acc[8 * j + 6] * invL, acc[8 * j + 7] * invL));
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int task = lane + 32 * k;
              const int rr = task >> 2, piece = task & 3;
              const int s = row0 + rr;
              const uint4 val = *reinterpret_cast<const uint4*>(xp + rr * XPOSE_PITCH + piece * 16);
              const long long oi = ((static_cast<long long>(b) * p.sched.Sq + s) * p.H + h) * HEAD_DIM + g * 32 + piece * 8;
              if (s < p.sched.Sq && in_bounds(oi + 7, p.out_elems, p.status))
                *reinterpret_cast<uint4*>(p.out + oi) = val;
            }
            __syncwarp();
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

template <class P, bool F8>
static cudaError_t prepare_kernel() {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    // the warpgroup register split assumes exactly LAUNCH_REGS registers per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, chunk_attn_kernel<P, F8>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(chunk_attn_kernel<P, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  return cudaSuccess;
}

static void fill_params(AttnParams& p, const AttnLaunch& a) {
  p.tm_q = a.tm_q;
  p.tm_k = a.tm_k;
  p.tm_v = a.tm_v;
  p.tm_ck = a.tm_ck;
  p.tm_cv = a.tm_cv;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.ws = a.ws;
  p.counters = a.counters;
  p.status = a.status;
  p.out_elems = a.out_elems;
  p.ws_slots = a.ws_slots;
  p.n_counters = a.n_counters;
  p.rope = a.rope;
  p.geom = a.geom;
  p.sched = a.sched;
  p.B = a.B;
  p.H = a.H;
  p.n_qg = a.n_qg;
  p.rope_q = a.rope_q;
  p.rope_k = a.rope_k;
  p.stage_ok = a.stage_ok;
  p.stage_t0 = a.stage_t0;
  p.stage_nt = a.stage_nt;
  p.W = static_cast<unsigned>(a.W);
  p.G = a.grid;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(HEAD_DIM)) *
                                    a.qk_scale);
}

template <bool F8>
static cudaError_t launch_variant(const AttnLaunch& a, cudaStream_t stream) {
  // the plain split computes c * W / G in 32 bits; past that the ranges go explicitly
  if (a.waves > 0 || a.W * (a.grid + 1LL) >= (1LL << 31)) {
    cudaError_t e = prepare_kernel<AttnParamsWaves, F8>();
    if (e != cudaSuccess) return e;
    AttnParamsWaves p;
    fill_params(p, a);
    p.waves = a.waves;
    for (int c = 0; c <= a.grid; ++c) p.tb[c] = a.tb[c];
    chunk_attn_kernel<AttnParamsWaves, F8><<<a.grid, NTHREADS, SMEM_BYTES, stream>>>(p);
  } else {
    cudaError_t e = prepare_kernel<AttnParams, F8>();
    if (e != cudaSuccess) return e;
    AttnParams p;
    fill_params(p, a);
    chunk_attn_kernel<AttnParams, F8><<<a.grid, NTHREADS, SMEM_BYTES, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream) {
  // E4M3 operands arrive rotated: the kernel would not rotate them
  if (a.e4m3 && (a.rope_q || a.rope_k)) return cudaErrorInvalidValue;
  return a.e4m3 ? launch_variant<true>(a, stream) : launch_variant<false>(a, stream);
}

}  // namespace dz
