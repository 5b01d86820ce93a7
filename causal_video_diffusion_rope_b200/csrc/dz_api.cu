// Host side of the C ABI declared in include/dz.h: argument checks, rotary
// tables, TMA tensor maps, the work split and the kernel launches.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/dz.h"
#include "dz_ops.cuh"

struct dz_attn {
  int device;
  int num_sms;
  dz_attn_desc desc;
  float2* rope_tab;
  int off_t, off_h, off_w;
  float* ws;           // 2 partial slots per CTA of the persistent grid
  int* counters;       // one per (batch, head, query group, Q tile)
  size_t n_counters;
  int* status;         // device status word
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  void* rot_ws;        // rotated q and k of teacher-forcing / prefill calls (or null)
  int rot_tokens;      // query tokens per batch item rot_ws holds
};

namespace {

using dz::cdiv;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// With DZ_DEBUG set in the environment, failing CUDA calls are reported on stderr.
bool debug_on() {
  static const bool on = std::getenv("DZ_DEBUG") != nullptr;
  return on;
}

dz_status cuda_status(cudaError_t e, const char* where = "") {
  if (e == cudaSuccess) return DZ_OK;
  if (debug_on()) std::fprintf(stderr, "[dz] %s: %s\n", where, cudaGetErrorString(e));
  return DZ_ERR_CUDA;
}

// 4-D view [B][rows][H][128] of a bf16 BSHD buffer whose batch stride is
// `rows_alloc` tokens; 64 x 1 x 128 x 1 boxes with 128-byte swizzle.  With `bytes`,
// the buffer holds one-byte (E4M3) elements and the boxes are 128 x 1 x 128 x 1.
dz_status make_map(const dz_attn* a, CUtensorMap* m, const void* base, int B, int rows,
                   int rows_alloc, int H, bool bytes = false) {
  const cuuint64_t esize = bytes ? 1 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(dz::HEAD_DIM), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(B)};
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(H) * dz::HEAD_DIM * esize;
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(dz::HEAD_DIM) * esize, row_bytes,
                                 row_bytes * static_cast<cuuint64_t>(rows_alloc)};
  const cuuint32_t box[4] = {bytes ? 128u : 64u, 1, static_cast<cuuint32_t>(dz::TILE_N), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = a->encode(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                         4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "[dz] cuTensorMapEncodeTiled failed (%d): dims %llu %llu %llu %llu\n",
                 static_cast<int>(r), static_cast<unsigned long long>(dims[0]),
                 static_cast<unsigned long long>(dims[1]), static_cast<unsigned long long>(dims[2]),
                 static_cast<unsigned long long>(dims[3]));
  return r == CUDA_SUCCESS ? DZ_OK : DZ_ERR_CUDA;
}

dz_status check_geom(const dz_chunk_layout* l) {
  if (l->frames_per_chunk < 1 || l->grid_h < 1 || l->grid_w < 1 || l->n_action < 0 ||
      l->t_offset < 0 || l->num_chunks < 0 || l->batch < 1)
    return DZ_ERR_INVALID_ARG;
  const long long L = static_cast<long long>(l->frames_per_chunk) * l->grid_h * l->grid_w +
                      l->n_action;
  if (L > (1 << 24)) return DZ_ERR_SHAPE;
  return DZ_OK;
}

dz::ChunkGeom geom_of(const dz_chunk_layout* l) {
  dz::ChunkGeom g;
  g.F = l->frames_per_chunk;
  g.gh = l->grid_h;
  g.gw = l->grid_w;
  g.L = l->frames_per_chunk * l->grid_h * l->grid_w + l->n_action;
  g.t_offset = l->t_offset;
  return g;
}

dz::RopeTables tables_of(const dz_attn* a) {
  dz::RopeTables r;
  r.tab = a->rope_tab;
  r.off_t = a->off_t;
  r.off_h = a->off_h;
  r.off_w = a->off_w;
  r.pt = a->desc.rope_pairs_t;
  r.ph = a->desc.rope_pairs_h;
  r.pw = a->desc.rope_pairs_w;
  r.n = a->off_w + a->desc.max_pos_w * a->desc.rope_pairs_w;
  return r;
}

// Chunks [first, last] of `g` must lie inside the rotary tables.
dz_status check_positions(const dz_attn* a, const dz::ChunkGeom& g, long long first_chunk,
                          long long last_chunk) {
  if (last_chunk < first_chunk) return DZ_OK;
  const long long t_max = g.t_offset + last_chunk * g.F + g.F - 1;
  if (t_max >= a->desc.max_pos_t || g.gh > a->desc.max_pos_h || g.gw > a->desc.max_pos_w)
    return DZ_ERR_SHAPE;
  return DZ_OK;
}

#ifdef DZ_TEST_HOOKS
// Test builds only (libdz_test.so): every attention call first fills its split
// counters with this value (0 = off).  A value with zero low half and a nonzero high
// half lets the pieces of a split unit count their arrivals as usual, while the
// merging piece's wait for the others' publications can never complete, so the
// bounded wait runs out and the call reports DZ_ERR_TIMEOUT.
int g_test_counter_fill = 0;
// Elements taken off the attention output's extent (dz_test_shrink_out), and the index
// faults of the bounds-checked kernels counted on the host (dz_test_bounds_faults).
long long g_test_out_shrink = 0;
long long g_test_bounds_faults = 0;
#endif

// Status of a nonzero device status word: an index fault of the bounds-checked build
// takes precedence over a wait that ran out (which it may have caused).
dz_status status_of_word(int word) {
#ifdef DZ_TEST_HOOKS
  if (word & dz::DZ_DEV_BOUNDS) ++g_test_bounds_faults;
#endif
  return (word & dz::DZ_DEV_BOUNDS) ? DZ_ERR_BOUNDS : DZ_ERR_TIMEOUT;
}


}  // namespace

namespace dz {

// Work split of an attention call over at most num_sms CTAs.
//  * One CTA per unit (no split) when the units fit the SMs and splitting would not
//    shorten the longest CTA by more than its merge costs.
//  * Otherwise `waves` rounds of whole units first, unit c + k * grid going to CTA c
//    (head-major order: the CTAs that run together work on the same few heads, whose
//    keys then come from L2), used when there is at least one full wave and the rest
//    is at least half a wave and no CTA's whole units exceed its balanced share; then
//    the remaining units' key tiles, cut into one contiguous range per CTA so that
//    every CTA ends up with the same estimated work (tiles plus a start-up cost per
//    whole unit).  A unit whose tiles fall in several ranges is merged from pieces.
void plan_schedule(AttnLaunch& a, const int* T, int n_qg, long long bh_count, int num_sms) {
  const long long units = bh_count * n_qg;
  long long per_bh = 0;
  int t_max = 0;
  for (int qg = 0; qg < n_qg; ++qg) {
    per_bh += T[qg];
    if (T[qg] > t_max) t_max = T[qg];
  }
  const long long W = per_bh * bh_count;
  a.W = W;
  // Units of equal size (decode, cross-attention, one query group per head) are
  // already whole in the plain contiguous split; only ragged ones use waves.
  const bool uniform = t_max * n_qg == per_bh;
  const int sms = num_sms < MAX_GRID ? num_sms : MAX_GRID;
  const long long split_tiles = (W + sms - 1) / sms;
  if (units <= sms && t_max <= split_tiles + SPLIT_OVERHEAD_TILES) {
    a.grid = static_cast<int>(units);
    a.waves = uniform ? 0 : 1;
    for (int c = 0; c <= a.grid; ++c)  // one unit per CTA, no tail
      a.tb[c] = static_cast<unsigned>(uniform ? c * W / a.grid : W);
    return;
  }
  const int G = static_cast<int>(W < sms ? W : sms);
  a.grid = G;
  int waves = 0;
  std::vector<double> R(G, 0.0);
  double target = static_cast<double>(W) / G;
  for (long long k = uniform ? 0 : units / G; k >= 1; --k) {
    if (units - k * G < G / 2) continue;
    std::vector<double> r(G, 0.0);
    long long wave_tiles = 0;
    for (long long u = 0; u < k * G; ++u) {
      const int t = T[u % n_qg];
      wave_tiles += t;
      r[u % G] += t + UNIT_SWITCH_TILES;
    }
    double tot = static_cast<double>(W - wave_tiles), rmax = 0.0;
    for (int c = 0; c < G; ++c) {
      tot += r[c];
      if (r[c] > rmax) rmax = r[c];
    }
    if (rmax <= tot / G) {
      waves = static_cast<int>(k);
      R = r;
      target = tot / G;
      break;
    }
  }
  a.waves = waves;
  long long P0 = 0;  // flattened position of the first unit of the tail
  for (long long u = 0; u < static_cast<long long>(waves) * G; ++u) P0 += T[u % n_qg];
  const long long tail = W - P0;
  a.tb[0] = static_cast<unsigned>(P0);
  if (waves == 0) {
    for (int c = 1; c <= G; ++c) a.tb[c] = static_cast<unsigned>(c * W / G);
  } else {
    double sum = 0.0;
    for (int c = 0; c < G; ++c) sum += target - R[c] > 0.0 ? target - R[c] : 0.0;
    double cum = 0.0;
    for (int c = 0; c < G; ++c) {
      cum += (target - R[c] > 0.0 ? target - R[c] : 0.0) * (static_cast<double>(tail) / sum);
      long long b = P0 + static_cast<long long>(cum);
      if (b > W) b = W;
      a.tb[c + 1] = static_cast<unsigned>(b);
    }
    a.tb[G] = static_cast<unsigned>(W);
  }
}

}  // namespace dz

extern "C" {

#ifdef DZ_TEST_HOOKS
void dz_test_fill_split_counters(int32_t value) { g_test_counter_fill = value; }

// Takes n elements off the output extent the next attention launches are given, so
// that the bounds-checked build's store checks fail for the last n elements.
void dz_test_shrink_out(int64_t n) { g_test_out_shrink = n; }

// Index faults seen by dz_attn_sync_status or dz_attn_destroy since the last call.
int64_t dz_test_bounds_faults(void) {
  const long long n = g_test_bounds_faults;
  g_test_bounds_faults = 0;
  return n;
}

// The work split of an attention call for `bh_count` (batch, head) pairs whose query
// groups have tiles[0 .. n_qg) key tiles each, over at most num_sms CTAs: writes the
// grid, the number of whole-unit waves and the tail ranges (grid + 1 entries of tb).
int32_t dz_test_plan_schedule(const int32_t* tiles, int32_t n_qg, int64_t bh_count,
                              int32_t num_sms, int32_t* grid, int32_t* waves, uint32_t* tb) {
  static dz::AttnLaunch a;
  dz::plan_schedule(a, tiles, n_qg, bh_count, num_sms);
  *grid = a.grid;
  *waves = a.waves;
  for (int c = 0; c <= a.grid; ++c) tb[c] = a.tb[c];
  return 0;
}
#endif

const char* dz_status_string(dz_status s) {
  switch (s) {
    case DZ_OK: return "ok";
    case DZ_ERR_INVALID_ARG: return "invalid argument";
    case DZ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case DZ_ERR_SHAPE: return "unsupported shape";
    case DZ_ERR_CAPACITY: return "capacity exceeded";
    case DZ_ERR_CUDA: return "CUDA error";
    case DZ_ERR_UNSUPPORTED: return "unsupported";
    case DZ_ERR_TIMEOUT: return "device wait timed out";
    case DZ_ERR_BOUNDS: return "device index check failed";
  }
  return "unknown status";
}

dz_status dz_attn_create(dz_attn_t* out, const dz_attn_desc* d) {
  if (!out || !d) return DZ_ERR_INVALID_ARG;
  *out = nullptr;
  if (d->head_dim != dz::HEAD_DIM) return DZ_ERR_SHAPE;
  if (d->num_heads < 1 || d->num_heads > 256) return DZ_ERR_SHAPE;
  if (d->rope_pairs_t < 0 || d->rope_pairs_h < 0 || d->rope_pairs_w < 0 ||
      d->rope_pairs_t + d->rope_pairs_h + d->rope_pairs_w != dz::HEAD_DIM / 2)
    return DZ_ERR_SHAPE;
  if (!(d->rope_base > 1.0) || !std::isfinite(d->rope_base)) return DZ_ERR_SHAPE;
  if (d->max_batch < 1 || d->max_q_tokens < 1 || d->max_pos_t < 1 || d->max_pos_h < 1 ||
      d->max_pos_w < 1 || d->prerotate_tokens < 0)
    return DZ_ERR_SHAPE;
  if (cdiv(d->max_q_tokens, dz::Q_GROUP) > dz::MAX_Q_GROUPS) return DZ_ERR_CAPACITY;
  if (static_cast<long long>(d->max_pos_t) * d->rope_pairs_t +
          static_cast<long long>(d->max_pos_h) * d->rope_pairs_h +
          static_cast<long long>(d->max_pos_w) * d->rope_pairs_w > (1ll << 28))
    return DZ_ERR_CAPACITY;

  dz_attn* a = new (std::nothrow) dz_attn();
  if (!a) return DZ_ERR_CUDA;
  a->desc = *d;
  if (cudaGetDevice(&a->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&a->num_sms, cudaDevAttrMultiProcessorCount, a->device) !=
          cudaSuccess) {
    delete a;
    return DZ_ERR_CUDA;
  }
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn) {
    delete a;
    return DZ_ERR_CUDA;
  }
  a->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);

  // rotary tables, built in double and stored as float (cos, sin)
  const int pt = d->rope_pairs_t, ph = d->rope_pairs_h, pw = d->rope_pairs_w;
  a->off_t = 0;
  a->off_h = d->max_pos_t * pt;
  a->off_w = a->off_h + d->max_pos_h * ph;
  const size_t n_tab = static_cast<size_t>(a->off_w) + static_cast<size_t>(d->max_pos_w) * pw;
  std::vector<float2> tab(n_tab > 0 ? n_tab : 1);
  auto fill = [&](int off, int npos, int npairs) {
    for (int j = 0; j < npairs; ++j) {
      const double omega = std::pow(d->rope_base, -2.0 * j / (2.0 * npairs));
      for (int p = 0; p < npos; ++p) {
        const double th = static_cast<double>(p) * omega;
        tab[off + static_cast<size_t>(p) * npairs + j] =
            make_float2(static_cast<float>(std::cos(th)), static_cast<float>(std::sin(th)));
      }
    }
  };
  fill(a->off_t, d->max_pos_t, pt);
  fill(a->off_h, d->max_pos_h, ph);
  fill(a->off_w, d->max_pos_w, pw);

  const int n_qg_max = cdiv(d->max_q_tokens, dz::Q_GROUP);
  a->n_counters = static_cast<size_t>(d->max_batch) * d->num_heads * n_qg_max * dz::Q_TILES;
  const size_t ws_floats = 2ull * a->num_sms * dz::PART_FLOATS;
  cudaError_t e = cudaMalloc(&a->rope_tab, tab.size() * sizeof(float2));
  if (e == cudaSuccess) e = cudaMalloc(&a->ws, ws_floats * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc(&a->counters, a->n_counters * sizeof(int));
  if (e == cudaSuccess) e = cudaMalloc(&a->status, sizeof(int));
  a->rot_ws = nullptr;
  a->rot_tokens = 0;
  if (e == cudaSuccess && d->prerotate_tokens > 0) {
    const size_t bytes = 2ull * d->max_batch * d->prerotate_tokens * d->num_heads * dz::HEAD_DIM * 2;
    e = cudaMalloc(&a->rot_ws, bytes);
    if (e == cudaSuccess) a->rot_tokens = d->prerotate_tokens;
  }
  if (e == cudaSuccess)
    e = cudaMemcpy(a->rope_tab, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(a->counters, 0, a->n_counters * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(a->status, 0, sizeof(int));
  // the copy and the memsets may return before they have landed; the handle's
  // calls run on other streams
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(a->rope_tab);
    cudaFree(a->ws);
    cudaFree(a->counters);
    cudaFree(a->status);
    cudaFree(a->rot_ws);
    delete a;
    return DZ_ERR_CUDA;
  }
  *out = a;
  return DZ_OK;
}

dz_status dz_attn_destroy(dz_attn_t a) {
  if (!a) return DZ_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
#ifdef DZ_TEST_HOOKS
  // an index fault that no status read reported is still counted
  int word = 0;
  if (e == cudaSuccess && cudaMemcpy(&word, a->status, sizeof(int), cudaMemcpyDeviceToHost) ==
                              cudaSuccess && (word & dz::DZ_DEV_BOUNDS))
    ++g_test_bounds_faults;
#endif
  cudaFree(a->rope_tab);
  cudaFree(a->ws);
  cudaFree(a->counters);
  cudaFree(a->status);
  cudaFree(a->rot_ws);
  delete a;
  return cuda_status(e);
}

static dz_status rope3d_call(dz_attn_t a, const void* x, void* y, int32_t B, int32_t S,
                             const dz_chunk_layout* layout, int32_t first_chunk, float e4m3_scale,
                             void* stream) {
  if (!a || !x || !y || !layout || B < 1 || S < 0 || first_chunk < 0) return DZ_ERR_INVALID_ARG;
  dz_chunk_layout l = *layout;
  l.batch = B;
  l.num_chunks = 0;
  dz_status st = check_geom(&l);
  if (st != DZ_OK) return st;
  if (!aligned16(x) || !aligned16(y)) return DZ_ERR_ALIGNMENT;
  if (S == 0) return DZ_OK;
  const dz::ChunkGeom g = geom_of(&l);
  st = check_positions(a, g, first_chunk, first_chunk + (S - 1) / g.L);
  if (st != DZ_OK) return st;
  return cuda_status(dz::launch_rope3d(x, y, B, S, a->desc.num_heads, g, first_chunk,
                                       tables_of(a), a->status, static_cast<cudaStream_t>(stream),
                                       nullptr, nullptr, 0, e4m3_scale),
                     "rope3d launch");
}

dz_status dz_rope3d(dz_attn_t a, const void* x, void* y, int32_t B, int32_t S,
                    const dz_chunk_layout* layout, int32_t first_chunk, void* stream) {
  return rope3d_call(a, x, y, B, S, layout, first_chunk, 0.f, stream);
}

dz_status dz_rope3d_e4m3(dz_attn_t a, const void* x, void* y8, int32_t B, int32_t S,
                         const dz_chunk_layout* layout, int32_t first_chunk, float scale,
                         void* stream) {
  if (!(scale > 0.f) || !std::isfinite(scale)) return DZ_ERR_INVALID_ARG;
  if (x == y8 && x != nullptr) return DZ_ERR_INVALID_ARG;  // one byte per element: no in-place
  return rope3d_call(a, x, y8, B, S, layout, first_chunk, scale, stream);
}

// The attention call; with lse != null (training form) it also writes each query
// row's log2-domain softmax normaliser.
// e4m3: null for bf16 q and k; else {q multiplier, k multiplier} of E4M3 q, k and
// cache k, which are then taken as rotated.
static dz_status attn_forward(dz_attn_t a, const void* q, const void* k, const void* v,
                              const dz_kvcache* cache, const dz_chunk_layout* l, void* out,
                              float* lse, void* stream, const float* e4m3 = nullptr) {
  if (!a || !q || !k || !v || !l || !out) return DZ_ERR_INVALID_ARG;
  if (e4m3) {
    for (int i = 0; i < 2; ++i)
      if (!(e4m3[i] > 0.f) || !std::isfinite(e4m3[i])) return DZ_ERR_INVALID_ARG;
    if (lse) return DZ_ERR_UNSUPPORTED;
  }
  // inputs already rotated: the flag is taken off a local copy of the layout
  const bool given_rotated = (l->mode & DZ_MODE_ROTATED) != 0 || e4m3 != nullptr;
  dz_chunk_layout l_plain = *l;
  l_plain.mode &= ~DZ_MODE_ROTATED;
  l = &l_plain;
  if (l->mode < DZ_MODE_DECODE || l->mode > DZ_MODE_CROSS) return DZ_ERR_INVALID_ARG;
  dz_status st = check_geom(l);
  if (st != DZ_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DZ_ERR_ALIGNMENT;
  if (l->batch > a->desc.max_batch) return DZ_ERR_CAPACITY;
  const int H = a->desc.num_heads;
  const dz::ChunkGeom g = geom_of(l);
  const long long L = g.L;
  long long Sq = 0, Sk = 0;
  int cache_len = 0;
  switch (l->mode) {
    case DZ_MODE_DECODE:
      Sq = Sk = L;
      if (cache) {
        if (!cache->k || !cache->v) return DZ_ERR_INVALID_ARG;
        if (!aligned16(cache->k) || !aligned16(cache->v)) return DZ_ERR_ALIGNMENT;
        if (cache->batch != l->batch || cache->len_tokens < 0 ||
            cache->len_tokens > cache->capacity_tokens)
          return DZ_ERR_INVALID_ARG;
        cache_len = cache->len_tokens;
      }
      break;
    case DZ_MODE_TEACHER_FORCING:
      if (cache) return DZ_ERR_INVALID_ARG;
      if (l->num_chunks < 1) return DZ_ERR_INVALID_ARG;
      Sq = Sk = 2 * L * l->num_chunks;
      break;
    case DZ_MODE_PREFILL:
      if (cache) return DZ_ERR_INVALID_ARG;
      if (l->num_chunks < 1) return DZ_ERR_INVALID_ARG;
      Sq = Sk = L * l->num_chunks;
      break;
    case DZ_MODE_CROSS:
      if (cache) return DZ_ERR_INVALID_ARG;
      if (l->num_chunks < 1 || l->kv_len < 1) return DZ_ERR_INVALID_ARG;
      Sq = L * l->num_chunks;
      Sk = l->kv_len;
      break;
  }
  if (Sq > a->desc.max_q_tokens) return DZ_ERR_CAPACITY;
  if (Sk > (1 << 28) || static_cast<long long>(cache_len) + Sk > (1 << 28)) return DZ_ERR_SHAPE;
  if (l->mode == DZ_MODE_DECODE) {
    st = check_positions(a, g, l->num_chunks, l->num_chunks);
  } else if (l->mode != DZ_MODE_CROSS) {
    st = check_positions(a, g, 0, l->num_chunks - 1);
  }
  if (st != DZ_OK) return st;

  dz::AttnLaunch p;
  std::memset(&p, 0, sizeof(p));
  p.e4m3 = e4m3 ? 1 : 0;
  p.qk_scale = e4m3 ? 1.0 / (static_cast<double>(e4m3[0]) * e4m3[1]) : 1.0;
  p.sched.mode = l->mode;
  p.sched.Sq = static_cast<int>(Sq);
  p.sched.Sk = static_cast<int>(Sk);
  p.sched.L = static_cast<int>(L);
  p.sched.N = l->num_chunks;
  p.sched.cache_len = cache_len;
  p.sched.nkc = cdiv(cache_len, dz::TILE_N);
  p.sched.nks = cdiv(static_cast<int>(Sk), dz::TILE_N);
  p.n_qg = cdiv(static_cast<int>(Sq), dz::Q_GROUP);
  if (p.n_qg > dz::MAX_Q_GROUPS) return DZ_ERR_CAPACITY;
  std::vector<int> tiles(p.n_qg);
  long long per_bh = 0;
  for (int qg = 0; qg < p.n_qg; ++qg) {
    tiles[qg] = dz::unit_tile_count(p.sched, qg);
    per_bh += tiles[qg];
  }
  const long long W = per_bh * l->batch * H;
  if (W <= 0) return DZ_ERR_SHAPE;
  // the kernel schedules key tiles with 32-bit arithmetic
  if (W >= (1LL << 31)) return DZ_ERR_UNSUPPORTED;
  dz::plan_schedule(p, tiles.data(), p.n_qg, static_cast<long long>(l->batch) * H, a->num_sms);
  p.B = l->batch;
  p.H = H;
  p.geom = g;
  p.rope = tables_of(a);
  p.rope_q = p.rope_k = (l->mode != DZ_MODE_CROSS && !given_rotated) ? 1 : 0;
  if (p.rope_q) {
    p.stage_t0 = g.t_offset + (l->mode == DZ_MODE_DECODE ? l->num_chunks * g.F : 0);
    p.stage_nt = (l->mode == DZ_MODE_DECODE ? 1 : l->num_chunks) * g.F;
    const long long n = static_cast<long long>(p.stage_nt) * a->desc.rope_pairs_t +
                        static_cast<long long>(g.gh) * a->desc.rope_pairs_h +
                        static_cast<long long>(g.gw) * a->desc.rope_pairs_w;
    p.stage_ok = n <= dz::ROPE_STAGE_MAX ? 1 : 0;
  }
  // with a workspace: rotate q and the call's own k once, before the attention kernel
  const void* q_att = q;
  const void* k_att = k;
  if (p.rope_q && a->rot_ws && Sq <= a->rot_tokens &&
      l->batch <= a->desc.max_batch) {
    const size_t elems = static_cast<size_t>(l->batch) * Sq * H * dz::HEAD_DIM;
    __nv_bfloat16* qr = static_cast<__nv_bfloat16*>(a->rot_ws);
    __nv_bfloat16* kr = qr + elems;
    const int period = l->mode == DZ_MODE_TEACHER_FORCING ? static_cast<int>(L * l->num_chunks) : 0;
    const int first = l->mode == DZ_MODE_DECODE ? l->num_chunks : 0;
    st = cuda_status(dz::launch_rope3d(q, qr, l->batch, static_cast<int>(Sq), H, g, first,
                                       tables_of(a), a->status, static_cast<cudaStream_t>(stream),
                                       k, kr, period),
                     "pre-rotation launch");
    if (st != DZ_OK) return st;
    q_att = qr;
    k_att = kr;
    p.rope_q = p.rope_k = 0;
    p.stage_ok = 0;
  }
  p.out = out;
  p.lse = lse;
  p.ws = a->ws;
  p.counters = a->counters;
  p.status = a->status;
  p.out_elems = static_cast<long long>(l->batch) * Sq * H * dz::HEAD_DIM;
  p.ws_slots = 2 * a->num_sms;
  p.n_counters = static_cast<long long>(a->n_counters);
#ifdef DZ_TEST_HOOKS
  p.out_elems -= g_test_out_shrink;
#endif

  const bool f8 = e4m3 != nullptr;
  st = make_map(a, &p.tm_q, q_att, l->batch, static_cast<int>(Sq), static_cast<int>(Sq), H, f8);
  if (st == DZ_OK)
    st = make_map(a, &p.tm_k, k_att, l->batch, static_cast<int>(Sk), static_cast<int>(Sk), H, f8);
  if (st == DZ_OK) st = make_map(a, &p.tm_v, v, l->batch, static_cast<int>(Sk), static_cast<int>(Sk), H);
  if (st == DZ_OK && cache_len > 0) {
    st = make_map(a, &p.tm_ck, cache->k, l->batch, cache_len, cache->capacity_tokens, H, f8);
    if (st == DZ_OK)
      st = make_map(a, &p.tm_cv, cache->v, l->batch, cache_len, cache->capacity_tokens, H);
  }
  if (st != DZ_OK) return st;
#ifdef DZ_TEST_HOOKS
  if (g_test_counter_fill != 0 &&
      dz::launch_fill_i32(a->counters, a->n_counters, g_test_counter_fill,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DZ_ERR_CUDA;
#endif
  return cuda_status(dz::launch_attention(p, static_cast<cudaStream_t>(stream)),
                     "attention launch");
}

dz_status dz_chunk_attn_forward(dz_attn_t a, const void* q, const void* k, const void* v,
                                const dz_kvcache* cache, const dz_chunk_layout* l, void* out,
                                void* stream) {
  return attn_forward(a, q, k, v, cache, l, out, nullptr, stream);
}

dz_status dz_chunk_attn_forward_e4m3(dz_attn_t a, const void* q8, const void* k8, const void* v,
                                     const dz_kvcache* cache, const dz_chunk_layout* l,
                                     float q_scale, float k_scale, void* out, void* stream) {
  const float sc[2] = {q_scale, k_scale};
  return attn_forward(a, q8, k8, v, cache, l, out, nullptr, stream, sc);
}

dz_status dz_quantize_e4m3(dz_attn_t a, const void* x, void* y, int64_t n, float scale,
                           void* stream) {
  if (!a || !x || !y || n < 0) return DZ_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return DZ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return DZ_ERR_ALIGNMENT;
  if (n == 0) return DZ_OK;
  return cuda_status(dz::launch_quantize_e4m3(static_cast<const __nv_bfloat16*>(x),
                                              static_cast<uint8_t*>(y), n, scale,
                                              static_cast<cudaStream_t>(stream)),
                     "quantize launch");
}

dz_status dz_chunk_attn_forward_lse(dz_attn_t a, const void* q, const void* k, const void* v,
                                    const dz_chunk_layout* l, void* out, void* lse,
                                    void* stream) {
  if (!l || !lse) return DZ_ERR_INVALID_ARG;
  const int mode = l->mode & ~DZ_MODE_ROTATED;
  if (mode != DZ_MODE_PREFILL && mode != DZ_MODE_TEACHER_FORCING) return DZ_ERR_UNSUPPORTED;
  if (!aligned16(lse)) return DZ_ERR_ALIGNMENT;
  return attn_forward(a, q, k, v, nullptr, l, out, static_cast<float*>(lse), stream);
}

dz_status dz_kvcache_append(dz_attn_t a, dz_kvcache* c, const void* k, const void* v,
                            void* stream) {
  if (!a || !c || !k || !v || !c->k || !c->v) return DZ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->chunk_len < 1 || c->len_tokens < 0 || c->capacity_tokens < 0 ||
      c->len_tokens > c->capacity_tokens)
    return DZ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(c->k) || !aligned16(c->v))
    return DZ_ERR_ALIGNMENT;
  if (static_cast<long long>(c->len_tokens) + c->chunk_len > c->capacity_tokens)
    return DZ_ERR_CAPACITY;
  cudaError_t e = dz::launch_kv_copy(k, v, c->k, c->v, c->batch, c->chunk_len, a->desc.num_heads,
                                     c->capacity_tokens, c->len_tokens, a->status,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return DZ_ERR_CUDA;
  c->len_tokens += c->chunk_len;
  return DZ_OK;
}

dz_status dz_kvcache_replace(dz_attn_t a, dz_kvcache* c, int32_t chunk_index, const void* k,
                             const void* v, void* stream) {
  if (!a || !c || !k || !v || !c->k || !c->v) return DZ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->chunk_len < 1 || c->len_tokens < 0 ||
      c->len_tokens > c->capacity_tokens || chunk_index < 0)
    return DZ_ERR_INVALID_ARG;
  if (static_cast<long long>(chunk_index + 1) * c->chunk_len > c->len_tokens)
    return DZ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(c->k) || !aligned16(c->v))
    return DZ_ERR_ALIGNMENT;
  return cuda_status(dz::launch_kv_copy(k, v, c->k, c->v, c->batch, c->chunk_len,
                                        a->desc.num_heads, c->capacity_tokens,
                                        chunk_index * c->chunk_len, a->status,
                                        static_cast<cudaStream_t>(stream)));
}

dz_status dz_qkv_rope(dz_attn_t a, const void* x, const void* w, int32_t B, int32_t S,
                      int32_t d_model, const dz_chunk_layout* l, int32_t first_chunk,
                      void* q_out, void* k_out, void* v_out, dz_kvcache* cache, void* stream) {
  if (!a || !x || !w || !l || !q_out || !k_out || !v_out) return DZ_ERR_INVALID_ARG;
  if (B < 1 || S < 1 || first_chunk < 0) return DZ_ERR_INVALID_ARG;
  dz_status st = check_geom(l);
  if (st != DZ_OK) return st;
  if (d_model < 64 || d_model % 64 != 0) return DZ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w) || !aligned16(q_out) || !aligned16(k_out) ||
      !aligned16(v_out))
    return DZ_ERR_ALIGNMENT;
  if (B > a->desc.max_batch) return DZ_ERR_CAPACITY;
  const int H = a->desc.num_heads;
  const long long M = static_cast<long long>(B) * S;
  const long long N = 3LL * H * dz::HEAD_DIM;
  if (M >= (1LL << 31) / dz::HEAD_DIM || N >= (1LL << 31)) return DZ_ERR_SHAPE;
  const dz::ChunkGeom g = geom_of(l);
  st = check_positions(a, g, first_chunk, first_chunk + (S - 1) / g.L);
  if (st != DZ_OK) return st;
  dz::QkvLaunch p = {};
  if (cache) {
    if (!cache->k || !cache->v) return DZ_ERR_INVALID_ARG;
    if (!aligned16(cache->k) || !aligned16(cache->v)) return DZ_ERR_ALIGNMENT;
    if (cache->batch != B || cache->chunk_len != S || cache->len_tokens < 0 ||
        cache->len_tokens > cache->capacity_tokens)
      return DZ_ERR_INVALID_ARG;
    if (static_cast<long long>(cache->len_tokens) + S > cache->capacity_tokens)
      return DZ_ERR_CAPACITY;
    p.ck = cache->k;
    p.cv = cache->v;
    p.cache_cap = cache->capacity_tokens;
    p.cache_row0 = cache->len_tokens;
    p.cache_batch = cache->batch;
  }
  // x as [M][d_model] with 64 x 256 boxes, w as [N][d_model] with 64 x bn boxes
  p.bn = dz::qkv_tile_n(M, N, a->num_sms);
  auto map2d = [&](CUtensorMap* m, const void* base, long long rows, int box_rows) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d_model), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d_model) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = a->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                                 dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DZ_OK : DZ_ERR_CUDA;
  };
  st = map2d(&p.tm_x, x, M, 256);
  if (st == DZ_OK) st = map2d(&p.tm_w, w, N, p.bn);
  if (st != DZ_OK) return st;
  p.q = q_out;
  p.k = k_out;
  p.v = v_out;
  p.M = static_cast<int>(M);
  p.S = S;
  p.H = H;
  p.K = d_model;
  p.rope = tables_of(a);
  p.geom = g;
  p.first_chunk = first_chunk;
  p.stage_t0 = g.t_offset + first_chunk * g.F;
  p.stage_nt = ((S - 1) / g.L + 1) * g.F;
  p.stage_ok = (static_cast<long long>(p.stage_nt) * a->desc.rope_pairs_t +
                    static_cast<long long>(g.gh) * a->desc.rope_pairs_h +
                    static_cast<long long>(g.gw) * a->desc.rope_pairs_w <=
                dz::QKV_ROPE_STAGE_MAX)
                   ? 1
                   : 0;
  p.status = a->status;
  p.num_sms = a->num_sms;
  st = cuda_status(dz::launch_qkv_rope(p, static_cast<cudaStream_t>(stream)), "qkv launch");
  if (st != DZ_OK) return st;
  if (cache) cache->len_tokens += S;
  return DZ_OK;
}

dz_status dz_chunk_attn_backward(dz_attn_t a, const void* q, const void* k, const void* v,
                                 const void* out, const void* dout, const void* lse,
                                 const dz_chunk_layout* l, void* dq, void* dk, void* dv,
                                 void* stream) {
  if (!a || !q || !k || !v || !out || !dout || !lse || !l || !dq || !dk || !dv)
    return DZ_ERR_INVALID_ARG;
  if (l->mode != DZ_MODE_PREFILL && l->mode != DZ_MODE_TEACHER_FORCING) return DZ_ERR_UNSUPPORTED;
  dz_status st = check_geom(l);
  if (st != DZ_OK) return st;
  if (l->num_chunks < 1) return DZ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return DZ_ERR_ALIGNMENT;
  if (l->batch > a->desc.max_batch) return DZ_ERR_CAPACITY;
  const int H = a->desc.num_heads;
  const dz::ChunkGeom g = geom_of(l);
  const long long S = (l->mode == DZ_MODE_TEACHER_FORCING ? 2LL : 1LL) * g.L * l->num_chunks;
  if (S > a->desc.max_q_tokens) return DZ_ERR_CAPACITY;
  // the rotated q, k go to the handle's rotation workspace and D to its split workspace
  if (!a->rot_ws || S > a->rot_tokens) return DZ_ERR_CAPACITY;
  const size_t ws_floats = 2ull * a->num_sms * dz::PART_FLOATS;
  if (static_cast<size_t>(l->batch) * H * S > ws_floats) return DZ_ERR_CAPACITY;
  st = check_positions(a, g, 0, l->num_chunks - 1);
  if (st != DZ_OK) return st;
  const size_t elems = static_cast<size_t>(l->batch) * S * H * dz::HEAD_DIM;
  __nv_bfloat16* qr = static_cast<__nv_bfloat16*>(a->rot_ws);
  __nv_bfloat16* kr = qr + elems;
  const int period = l->mode == DZ_MODE_TEACHER_FORCING ? g.L * l->num_chunks : 0;
  st = cuda_status(dz::launch_rope3d(q, qr, l->batch, static_cast<int>(S), H, g, 0, tables_of(a),
                                     a->status, static_cast<cudaStream_t>(stream), k, kr, period),
                   "backward rotation launch");
  if (st != DZ_OK) return st;
  dz::BwdLaunch p;
  st = make_map(a, &p.tm_q, qr, l->batch, static_cast<int>(S), static_cast<int>(S), H);
  if (st == DZ_OK) st = make_map(a, &p.tm_k, kr, l->batch, static_cast<int>(S), static_cast<int>(S), H);
  if (st == DZ_OK) st = make_map(a, &p.tm_v, v, l->batch, static_cast<int>(S), static_cast<int>(S), H);
  if (st == DZ_OK) st = make_map(a, &p.tm_do, dout, l->batch, static_cast<int>(S), static_cast<int>(S), H);
  if (st != DZ_OK) return st;
  p.out = out;
  p.dout = dout;
  p.lse = static_cast<const float*>(lse);
  p.dd = a->ws;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.rope = tables_of(a);
  p.geom = g;
  p.mode = l->mode;
  p.N = l->num_chunks;
  p.S = static_cast<int>(S);
  p.B = l->batch;
  p.H = H;
  p.status = a->status;
  return cuda_status(dz::launch_backward(p, static_cast<cudaStream_t>(stream)), "backward launch");
}

static dz_status noalloc_sync_status(void* stream);

dz_status dz_attn_sync_status(dz_attn_t a, void* stream) {
  if (!a) return noalloc_sync_status(stream);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DZ_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, a->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DZ_ERR_CUDA;
  if (word != 0) {
    // a kernel gave up mid-call: clear the word and the split counters it may have left
    if (cudaMemset(a->status, 0, sizeof(int)) != cudaSuccess ||
        cudaMemset(a->counters, 0, a->n_counters * sizeof(int)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
      return DZ_ERR_CUDA;
    return status_of_word(word);
  }
  return DZ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Attention without any allocation, for callers that cannot call cudaMalloc.
//
// The scratch memory the attention kernel needs (fp32 partial results of split
// work units, the split counters and a status word) lives in one file-scope
// static device array, and the rotary tables in a second one; both are created
// with the module, so every GPU that loads this library holds them until the
// process exits.  On host code the array names are host-side stand-ins, not
// device addresses: their device addresses are looked up once per device with
// cudaGetSymbolAddress, with that device current.
// ---------------------------------------------------------------------------
namespace {

constexpr int NOALLOC_SLOTS = 126;                 // partial-result slots (2 per CTA)
constexpr size_t NOALLOC_WS_BYTES = NOALLOC_SLOTS * dz::PART_FLOATS * sizeof(float);
constexpr size_t NOALLOC_COUNTERS = 65536;         // split counters
constexpr size_t NOALLOC_SCRATCH_BYTES = NOALLOC_WS_BYTES + NOALLOC_COUNTERS * sizeof(int) + 256;
constexpr size_t NOALLOC_ROPE_ENTRIES = 294912;    // (cos, sin) pairs of the rotary tables

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];
static __device__ __align__(256) float2 g_noalloc_rope[NOALLOC_ROPE_ENTRIES];

struct NoallocDevice {
  bool ready = false;
  int num_sms = 0;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  float2* rope = nullptr;            // device address of g_noalloc_rope
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  bool tables = false;               // rotary tables hold `rot` below
  double base = 0.0;
  int pt = 0, ph = 0, pw = 0, mt = 0, mh = 0, mw = 0;
};
NoallocDevice g_noalloc[64];
std::mutex g_noalloc_mu;

}  // namespace

extern "C" dz_status dz_chunk_attn_forward_noalloc(const dz_attn_desc* d, const void* q,
                                                   const void* k, const void* v,
                                                   const dz_kvcache* cache,
                                                   const dz_chunk_layout* layout, void* out,
                                                   void* stream) {
  if (!d || !layout) return DZ_ERR_INVALID_ARG;
  if (d->head_dim != dz::HEAD_DIM || d->num_heads < 1 || d->num_heads > 256) return DZ_ERR_SHAPE;
  if (d->rope_pairs_t < 0 || d->rope_pairs_h < 0 || d->rope_pairs_w < 0 ||
      d->rope_pairs_t + d->rope_pairs_h + d->rope_pairs_w != dz::HEAD_DIM / 2)
    return DZ_ERR_SHAPE;
  if (!(d->rope_base > 1.0) || !std::isfinite(d->rope_base)) return DZ_ERR_SHAPE;
  if (d->max_batch < 1 || d->max_q_tokens < 1 || d->max_pos_t < 1 || d->max_pos_h < 1 ||
      d->max_pos_w < 1)
    return DZ_ERR_SHAPE;
  // sizes beyond what the static arrays hold are rejected
  const long long n_qg_max = cdiv(d->max_q_tokens, dz::Q_GROUP);
  if (n_qg_max > dz::MAX_Q_GROUPS ||
      static_cast<long long>(d->max_batch) * d->num_heads * n_qg_max * dz::Q_TILES >
          static_cast<long long>(NOALLOC_COUNTERS)) {
    if (debug_on())
      std::fprintf(stderr, "[dz] noalloc: batch x heads x query groups exceeds %zu counters\n",
                   NOALLOC_COUNTERS);
    return DZ_ERR_CAPACITY;
  }
  const long long n_tab = static_cast<long long>(d->max_pos_t) * d->rope_pairs_t +
                          static_cast<long long>(d->max_pos_h) * d->rope_pairs_h +
                          static_cast<long long>(d->max_pos_w) * d->rope_pairs_w;
  if (n_tab > static_cast<long long>(NOALLOC_ROPE_ENTRIES)) {
    if (debug_on())
      std::fprintf(stderr, "[dz] noalloc: rotary tables need %lld entries, %zu available\n",
                   n_tab, NOALLOC_ROPE_ENTRIES);
    return DZ_ERR_CAPACITY;
  }

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DZ_ERR_CUDA;
  NoallocDevice& nd = g_noalloc[dev];
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!nd.ready) {
      // once per device, with that device current: device addresses of the arrays
      void* sp = nullptr;
      void* rp = nullptr;
      if (cudaGetSymbolAddress(&sp, g_noalloc_scratch) != cudaSuccess ||
          cudaGetSymbolAddress(&rp, g_noalloc_rope) != cudaSuccess)
        return DZ_ERR_CUDA;
      cudaDriverEntryPointQueryResult qr;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) !=
              cudaSuccess ||
          qr != cudaDriverEntryPointSuccess || !fn)
        return DZ_ERR_CUDA;
      if (cudaDeviceGetAttribute(&nd.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DZ_ERR_CUDA;
      nd.scratch = static_cast<unsigned char*>(sp);
      nd.rope = static_cast<float2*>(rp);
      nd.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      nd.ready = true;
    }
    if (!nd.tables || nd.base != d->rope_base || nd.pt != d->rope_pairs_t ||
        nd.ph != d->rope_pairs_h || nd.pw != d->rope_pairs_w || nd.mt != d->max_pos_t ||
        nd.mh != d->max_pos_h || nd.mw != d->max_pos_w) {
      // (re)build the rotary tables for this rotary configuration: a synchronous copy
      std::vector<float2> tab(static_cast<size_t>(n_tab));
      size_t off = 0;
      const int npos[3] = {d->max_pos_t, d->max_pos_h, d->max_pos_w};
      const int npairs[3] = {d->rope_pairs_t, d->rope_pairs_h, d->rope_pairs_w};
      for (int ax = 0; ax < 3; ++ax) {
        for (int j = 0; j < npairs[ax]; ++j) {
          const double omega = std::pow(d->rope_base, -2.0 * j / (2.0 * npairs[ax]));
          for (int pp = 0; pp < npos[ax]; ++pp) {
            const double th = static_cast<double>(pp) * omega;
            tab[off + static_cast<size_t>(pp) * npairs[ax] + j] =
                make_float2(static_cast<float>(std::cos(th)), static_cast<float>(std::sin(th)));
          }
        }
        off += static_cast<size_t>(npos[ax]) * npairs[ax];
      }
      // earlier calls (on any stream) may still read the old tables: the device must
      // be idle before they are overwritten, and the new ones must have landed
      // before this call's kernels run
      if (cudaDeviceSynchronize() != cudaSuccess) return DZ_ERR_CUDA;
      if (!tab.empty() && (cudaMemcpy(nd.rope, tab.data(), tab.size() * sizeof(float2),
                                      cudaMemcpyHostToDevice) != cudaSuccess ||
                           cudaDeviceSynchronize() != cudaSuccess))
        return DZ_ERR_CUDA;
      nd.tables = true;
      nd.base = d->rope_base;
      nd.pt = d->rope_pairs_t;
      nd.ph = d->rope_pairs_h;
      nd.pw = d->rope_pairs_w;
      nd.mt = d->max_pos_t;
      nd.mh = d->max_pos_h;
      nd.mw = d->max_pos_w;
    }
  }

  // a handle-shaped view of the static memory; the grid is capped so that each
  // CTA's two partial-result slots fit in the static workspace
  dz_attn a;
  a.device = dev;
  a.num_sms = nd.num_sms < NOALLOC_SLOTS / 2 ? nd.num_sms : NOALLOC_SLOTS / 2;
  a.desc = *d;
  a.rope_tab = nd.rope;
  a.off_t = 0;
  a.off_h = d->max_pos_t * d->rope_pairs_t;
  a.off_w = a.off_h + d->max_pos_h * d->rope_pairs_h;
  a.ws = reinterpret_cast<float*>(nd.scratch);
  a.counters = reinterpret_cast<int*>(nd.scratch + NOALLOC_WS_BYTES);
  a.n_counters = static_cast<size_t>(d->max_batch) * d->num_heads * n_qg_max * dz::Q_TILES;
  a.status = reinterpret_cast<int*>(nd.scratch + NOALLOC_WS_BYTES + NOALLOC_COUNTERS * sizeof(int));
  a.encode = nd.encode;
  a.rot_ws = nullptr;  // no pre-rotation workspace: rotation stays inside the kernel
  a.rot_tokens = 0;
  // the split counters must start at zero (a previous call that gave up may have left
  // them set); cleared on the caller's stream.  The status word keeps a timeout until
  // dz_attn_sync_status(NULL, stream) reads and clears it.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a.counters, 0, a.n_counters * sizeof(int), st) != cudaSuccess)
    return DZ_ERR_CUDA;
  return dz_chunk_attn_forward(&a, q, k, v, cache, layout, out, stream);
}

// Status of the allocation-free calls on the current device (dz_attn_sync_status
// with a NULL handle).
static dz_status noalloc_sync_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DZ_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DZ_ERR_CUDA;
  unsigned char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc[dev].ready) return DZ_OK;  // no allocation-free call on this device yet
    scratch = g_noalloc[dev].scratch;
  }
  int* counters = reinterpret_cast<int*>(scratch + NOALLOC_WS_BYTES);
  int* status = reinterpret_cast<int*>(scratch + NOALLOC_WS_BYTES + NOALLOC_COUNTERS * sizeof(int));
  int word = 0;
  if (cudaMemcpy(&word, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DZ_ERR_CUDA;
  if (word == 0) return DZ_OK;
  if (cudaMemset(status, 0, sizeof(int)) != cudaSuccess ||
      cudaMemset(counters, 0, NOALLOC_COUNTERS * sizeof(int)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess)
    return DZ_ERR_CUDA;
  return status_of_word(word);
}
