// Internal declarations shared by the host API (dz_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace dz {

enum { MODE_DECODE = 0, MODE_TEACHER_FORCING = 1, MODE_PREFILL = 2, MODE_CROSS = 3 };

constexpr int HEAD_DIM = 128;
constexpr int TILE_M = 128;        // query rows per Q tile (TMEM lanes)
constexpr int TILE_N = 128;        // keys per K/V tile
constexpr int Q_TILES = 2;         // Q tiles per CTA (ping-pong between two softmax groups)
constexpr int Q_GROUP = TILE_M * Q_TILES;  // query rows per work unit
constexpr int MAX_Q_GROUPS = 512;  // per (batch, head); bounds the per-CTA prefix table
constexpr int MAX_GRID = 256;      // CTAs of one attention launch (the schedule is a kernel parameter)

// Status-word bit of the bounds-checked build: an index check failed (the access
// was skipped).  Bit 0 is a device wait that ran out (dz_ptx.cuh).
constexpr int DZ_DEV_BOUNDS = 2;

// Index check of the bounds-checked build (DZ_DEBUG_BOUNDS): whether element i of a
// buffer of n elements may be accessed.  A failed check records DZ_DEV_BOUNDS in the
// status word and the caller skips the access.  Other builds compile it away.
__device__ __forceinline__ bool in_bounds(long long i, long long n, int* status) {
#ifdef DZ_DEBUG_BOUNDS
  if (i >= 0 && i < n) return true;
  atomicOr(status, DZ_DEV_BOUNDS);
  return false;
#else
  (void)i;
  (void)n;
  (void)status;
  return true;
#endif
}

// Rotary tables: (cos, sin) as float2 for every (axis position, pair of that axis).
struct RopeTables {
  const float2* tab;
  int off_t, off_h, off_w;  // element offsets of the t, h and w tables
  int pt, ph, pw;           // pairs per axis
  int n;                    // entries of tab
};

// Token-to-position rule of a run of whole chunks (see dz.h): token s of the
// run sits at offset s % L of chunk first_chunk + s / L.
struct ChunkGeom {
  int L, F, gh, gw, t_offset;
};

__host__ __device__ __forceinline__ void token_pos(const ChunkGeom& g, int s, int first_chunk,
                                                   int& t, int& h, int& w) {
  const int n = first_chunk + s / g.L;
  const int o = s - (s / g.L) * g.L;
  const int per_frame = g.gh * g.gw;
  if (o < g.F * per_frame) {
    const int f = o / per_frame;
    const int rem = o - f * per_frame;
    t = g.t_offset + n * g.F + f;
    h = rem / g.gw;
    w = rem - h * g.gw;
  } else {
    t = g.t_offset + n * g.F;
    h = 0;
    w = 0;
  }
}

// Index into RopeTables::tab of pair j at position (t, h, w).
__device__ __forceinline__ int rope_index(const RopeTables& r, int j, int t, int h, int w) {
  const int pth = r.pt + r.ph;
  return j < r.pt ? r.off_t + t * r.pt + j
                  : (j < pth ? r.off_h + h * r.ph + (j - r.pt) : r.off_w + w * r.pw + (j - pth));
}

// rope_index checked against the table in the bounds-checked build (entry 0 when
// the check fails).
__device__ __forceinline__ int rope_index_checked(const RopeTables& r, int j, int t, int h, int w,
                                                  int* status) {
  const int i = rope_index(r, j, t, h, w);
  return in_bounds(i, r.n, status) ? i : 0;
}

// One rotated pair (two bf16 in a 32-bit word) in fp32, rounded to bf16.  Used
// by the standalone rotary kernel and the attention kernel's fused tile
// rotation alike, so both give identical bf16 results.
__device__ __forceinline__ uint32_t rope_pair(uint32_t xbits, float2 cs) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&xbits);
  const float x0 = __low2float(x), x1 = __high2float(x);
  const float y0 = __fmaf_rn(x0, cs.x, -__fmul_rn(x1, cs.y));
  const float y1 = __fmaf_rn(x0, cs.y, __fmul_rn(x1, cs.x));
  __nv_bfloat162 y = __floats2bfloat162_rn(y0, y1);
  return *reinterpret_cast<uint32_t*>(&y);
}

// ---------------------------------------------------------------------------
// Work decomposition of one attention call.
// A unit is (batch, head, query group of Q_GROUP rows).  Its key tiles (in the
// key-tile space of the call) are [0, e1) followed by [s2, e2), s2 >= e1.
// ---------------------------------------------------------------------------
struct SchedGeom {
  int mode;
  int Sq;         // query tokens per batch item
  int Sk;         // keys in the call's own k/v per batch item
  int L;          // chunk length
  int N;          // num_chunks
  int cache_len;  // DECODE: cached keys
  int nkc;        // DECODE: cache key tiles
  int nks;        // own key tiles
};

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ __forceinline__ void unit_tiles(const SchedGeom& g, int qg, int& e1, int& s2,
                                                    int& e2) {
  s2 = e2 = 0;
  if (g.mode == MODE_DECODE) {
    e1 = g.nkc + g.nks;
    s2 = e2 = e1;
    return;
  }
  if (g.mode == MODE_CROSS) {
    e1 = g.nks;
    s2 = e2 = e1;
    return;
  }
  const int q0 = qg * Q_GROUP;
  const int q1 = (q0 + Q_GROUP < g.Sq) ? q0 + Q_GROUP : g.Sq;
  const int c0 = q0 / g.L, c1 = (q1 - 1) / g.L;
  if (g.mode == MODE_PREFILL) {
    int x = (c1 + 1) * g.L;
    if (x > g.Sk) x = g.Sk;
    e1 = cdiv(x, TILE_N);
    s2 = e2 = e1;
    return;
  }
  // teacher forcing: clean chunks [0, N), noisy chunks [N, 2N)
  int x = 0;
  bool noisy = false;
  int y = 0, z = 0;
  if (c0 < g.N) {
    const int cc = c1 < g.N - 1 ? c1 : g.N - 1;
    x = (cc + 1) * g.L;
  }
  if (c1 >= g.N) {
    const int i0 = (c0 > g.N ? c0 : g.N) - g.N;
    const int i1 = c1 - g.N;
    if (i1 * g.L > x) x = i1 * g.L;
    y = (g.N + i0) * g.L;
    z = (g.N + i1 + 1) * g.L;
    noisy = true;
  }
  e1 = cdiv(x, TILE_N);
  if (noisy) {
    s2 = y / TILE_N;
    e2 = cdiv(z, TILE_N);
    if (s2 <= e1) {
      if (e2 > e1) e1 = e2;
      s2 = e2 = e1;
    }
  } else {
    s2 = e2 = e1;
  }
}

__host__ __device__ __forceinline__ int unit_tile_count(const SchedGeom& g, int qg) {
  int e1, s2, e2;
  unit_tiles(g, qg, e1, s2, e2);
  return e1 + (e2 - s2);
}

// ---------------------------------------------------------------------------
// Kernel launchers (defined in the .cu files; return cudaGetLastError()).
// ---------------------------------------------------------------------------
cudaError_t launch_kv_copy(const void* k, const void* v, void* ck, void* cv, int B, int rows,
                           int H, int cap, int dst_row0, int* status, cudaStream_t stream);
#ifdef DZ_TEST_HOOKS
// Test builds only: x[0:n] = value.
cudaError_t launch_fill_i32(int* x, size_t n, int value, cudaStream_t stream);
#endif

// Rotates x into y (and x1 into y1 when x1 is not null) for B x S tokens; with
// period > 0 token s is rotated at the position of token s % period.  With
// e4m3_scale > 0 the outputs are the E4M3 codes of the rotated bf16 values times
// e4m3_scale (one byte per element).  `status` receives the bounds-checked build's
// index faults.
cudaError_t launch_rope3d(const void* x, void* y, int B, int S, int H, const ChunkGeom& g,
                          int first_chunk, const RopeTables& r, int* status, cudaStream_t stream,
                          const void* x1 = nullptr, void* y1 = nullptr, int period = 0,
                          float e4m3_scale = 0.f);

// y[0:n] = E4M3 codes of x[0:n] * scale (round to nearest even, saturating at 448).
cudaError_t launch_quantize_e4m3(const __nv_bfloat16* x, uint8_t* y, long long n, float scale,
                                 cudaStream_t stream);

struct AttnLaunch {
  CUtensorMap tm_q, tm_k, tm_v, tm_ck, tm_cv;
  void* out;
  float* lse;  // null, or fp32 [B][H][Sq]: m + log2(l) of each query row's softmax
  float* ws;
  int* counters;
  int* status;
  // extents for the bounds-checked build: out elements (B * Sq * H * 128; lse has
  // a 128th of that), partial-result slots of ws, split counters
  long long out_elems;
  int ws_slots;
  long long n_counters;
  RopeTables rope;
  ChunkGeom geom;
  SchedGeom sched;
  int B, H;
  int n_qg;
  int rope_q, rope_k;
  // rotary-table rows the call needs (t in [stage_t0, stage_t0 + stage_nt), all h < gh,
  // all w < gw), copied to shared memory at kernel start when stage_ok
  int stage_ok, stage_t0, stage_nt;
  // Schedule over `grid` CTAs: `waves` rounds of whole units dealt round-robin (CTA c
  // takes unit c + k * grid of the head-major order), then CTA c takes the flattened
  // key tiles [tb[c], tb[c + 1]) of the remaining units, splitting units between CTAs.
  // With waves == 0, tb[c] = c * W / grid (W = all units' key tiles).
  long long W;
  int grid;
  int waves;
  unsigned tb[MAX_GRID + 1];
  // q and k (and cache k) are rotated E4M3 codes rather than bf16; the scores are
  // multiplied by qk_scale (1 / (q multiplier * k multiplier); 1 for bf16 operands)
  int e4m3;
  double qk_scale;
};

// Schedule of an attention call (see AttnLaunch): fills grid, waves and tb from the
// tile counts of the query groups of one (batch, head), `units_bh` groups each.
void plan_schedule(AttnLaunch& a, const int* tiles_per_qg, int n_qg, long long bh_count,
                   int num_sms);

// Cost of splitting a unit across CTAs (partial write, merge, extra Q loads), in
// key tiles: a call runs one unit per CTA unless splitting saves more than this.
constexpr int SPLIT_OVERHEAD_TILES = 10;
// Estimated cost of starting a unit (Q load, pipeline fill, epilogue), in key tiles,
// used to balance the whole units of the round-robin waves against the tail.
constexpr int UNIT_SWITCH_TILES = 2;

// Capacity (float2 entries) of the attention kernel's shared-memory rotary table.
constexpr int ROPE_STAGE_MAX = 1280;

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t stream);

// Workspace (in floats) one partial-result slot needs: Q_TILES * TILE_M rows of
// HEAD_DIM accumulators plus (m, l) per row.
constexpr size_t PART_FLOATS = static_cast<size_t>(Q_TILES) * TILE_M * (HEAD_DIM + 2);

}  // namespace dz
