// Bandwidth-bound kernels: KV-cache append/replace (a 16-byte vectorised
// copy), the standalone 3D rotary embedding and the E4M3 quantisation.
#include <cuda_fp8.h>

#include "dz_internal.cuh"
#include "dz_ptx.cuh"

namespace dz {

// ---------------------------------------------------------------------------
// KV-cache chunk copy.  One chunk of keys and values, bf16 [B][rows][H][128],
// is contiguous per batch item; in the cache [B][cap][H][128] it lands at rows
// [dst_row0, dst_row0 + rows).  blockIdx.y selects (tensor, batch item); each
// thread moves 4 independent 16-byte vectors per iteration (grid-stride).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kv_copy_kernel(const uint4* __restrict__ k,
                                                      const uint4* __restrict__ v,
                                                      uint4* __restrict__ ck,
                                                      uint4* __restrict__ cv, int B,
                                                      long long span_vecs, long long src_stride,
                                                      long long dst_stride, long long dst_off,
                                                      int* status) {
  const int which = blockIdx.y / B;  // 0 = keys, 1 = values
  const int b = blockIdx.y - which * B;
  const uint4* src = (which == 0 ? k : v) + static_cast<long long>(b) * src_stride;
  uint4* dst = (which == 0 ? ck : cv) + static_cast<long long>(b) * dst_stride + dst_off;
  const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
#ifdef DZ_DEBUG_BOUNDS
  // the destination rows must lie inside this batch item's cache rows
  if (!in_bounds(dst_off + span_vecs - 1, dst_stride, status)) return;
#else
  (void)status;
#endif
  for (; i + 3 * step < span_vecs; i += 4 * step) {
    const uint4 a0 = src[i], a1 = src[i + step], a2 = src[i + 2 * step], a3 = src[i + 3 * step];
    dst[i] = a0;
    dst[i + step] = a1;
    dst[i + 2 * step] = a2;
    dst[i + 3 * step] = a3;
  }
  for (; i < span_vecs; i += step) dst[i] = src[i];
}

cudaError_t launch_kv_copy(const void* k, const void* v, void* ck, void* cv, int B, int rows,
                           int H, int cap, int dst_row0, int* status, cudaStream_t stream) {
  const long long row_vecs = static_cast<long long>(H) * HEAD_DIM * 2 / 16;
  const long long span = row_vecs * rows;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // about 8 resident blocks of 256 threads per SM over the 2*B spans
  long long want = (static_cast<long long>(sms) * 8 + 2 * B - 1) / (2 * B);
  long long need = (span + 256 * 4 - 1) / (256 * 4);
  int gx = static_cast<int>(want < need ? want : need);
  if (gx < 1) gx = 1;
  dim3 grid(gx, 2 * B);
  kv_copy_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(ck),
      static_cast<uint4*>(cv), B, span, span, row_vecs * cap, row_vecs * dst_row0, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// 3D rotary embedding of whole tokens.  One block per token (b, s) of each of
// up to two tensors (blockIdx.y): its position is computed once, then the
// block's threads rotate the token's H*16 16-byte chunks.  A thread always
// handles the same 4 pairs (chunk index mod 16), so it reads its 4 (cos, sin)
// entries once and then streams one chunk per head, all loads of a thread
// issued before its stores.  With period > 0, token s takes the position of
// token s % period (the noisy half of a teacher-forcing sequence shares the
// clean half's positions).
// x and y may be the same buffer (in place): each thread reads and then writes
// the same 16 bytes, so they are not declared __restrict__.  With E4M3 output each
// rotated bf16 value is also quantised (times `scale`, as dz_quantize_e4m3 does) and
// a 16-byte chunk becomes 8 bytes.
// ---------------------------------------------------------------------------
constexpr int ROPE_BLOCK = 128;
constexpr int ROPE_UNROLL = 8;  // chunks per thread per pass: 64 heads with 128 threads

// Four bf16 values (two packed pairs) times scale, as E4M3 codes: the fp32 product,
// rounded to nearest even with magnitudes past 448 saturating.
__device__ __forceinline__ uint32_t e4m3x4(uint32_t lo2, uint32_t hi2, float scale) {
  const float2 a = make_float2(__fmul_rn(__uint_as_float(lo2 << 16), scale),
                               __fmul_rn(__uint_as_float(lo2 & 0xffff0000u), scale));
  const float2 b = make_float2(__fmul_rn(__uint_as_float(hi2 << 16), scale),
                               __fmul_rn(__uint_as_float(hi2 & 0xffff0000u), scale));
  const uint32_t pa = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
  const uint32_t pb = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
  return pa | (pb << 16);
}

template <bool E4M3>
__global__ void __launch_bounds__(ROPE_BLOCK) rope3d_kernel(const uint4* x0, void* y0,
                                                            const uint4* x1, void* y1, int S,
                                                            int H, ChunkGeom g, int first_chunk,
                                                            int period, RopeTables r, float scale,
                                                            int* status) {
  const long long token = blockIdx.x;  // b * S + s
  int s = static_cast<int>(token % S);
  if (period > 0) s %= period;
  int t, hh, w;
  token_pos(g, s, first_chunk, t, hh, w);
  const int nvec = H * (HEAD_DIM / 8);
  const uint4* src = (blockIdx.y == 0 ? x0 : x1) + token * nvec;
  void* dst_base = blockIdx.y == 0 ? y0 : y1;
  const int j0 = (threadIdx.x & 15) * 4;  // ROPE_BLOCK is a multiple of 16
  float2 cs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) cs[k] = __ldg(r.tab + rope_index_checked(r, j0 + k, t, hh, w, status));
  for (int i0 = threadIdx.x; i0 < nvec; i0 += ROPE_BLOCK * ROPE_UNROLL) {
    uint4 v[ROPE_UNROLL];
#pragma unroll
    for (int u = 0; u < ROPE_UNROLL; ++u) {
      const int i = i0 + u * ROPE_BLOCK;
      if (i < nvec) v[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < ROPE_UNROLL; ++u) {
      const int i = i0 + u * ROPE_BLOCK;
      if (i < nvec) {
        const uint4 o = make_uint4(rope_pair(v[u].x, cs[0]), rope_pair(v[u].y, cs[1]),
                                   rope_pair(v[u].z, cs[2]), rope_pair(v[u].w, cs[3]));
        if constexpr (E4M3)
          (static_cast<uint2*>(dst_base) + token * nvec)[i] =
              make_uint2(e4m3x4(o.x, o.y, scale), e4m3x4(o.z, o.w, scale));
        else
          (static_cast<uint4*>(dst_base) + token * nvec)[i] = o;
      }
    }
  }
}

cudaError_t launch_rope3d(const void* x, void* y, int B, int S, int H, const ChunkGeom& g,
                          int first_chunk, const RopeTables& r, int* status, cudaStream_t stream,
                          const void* x1, void* y1, int period, float e4m3_scale) {
  const long long tokens = static_cast<long long>(B) * S;
  if (tokens <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(tokens), x1 ? 2 : 1);
  if (e4m3_scale > 0.f)
    rope3d_kernel<true><<<grid, ROPE_BLOCK, 0, stream>>>(static_cast<const uint4*>(x), y,
                                                         static_cast<const uint4*>(x1), y1, S, H, g,
                                                         first_chunk, period, r, e4m3_scale, status);
  else
    rope3d_kernel<false><<<grid, ROPE_BLOCK, 0, stream>>>(static_cast<const uint4*>(x), y,
                                                          static_cast<const uint4*>(x1), y1, S, H, g,
                                                          first_chunk, period, r, 0.f, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// E4M3 quantisation: y[i] = E4M3(float(x[i]) * scale), rounded to nearest even with
// magnitudes past 448 saturating (the FP8 operands of the attention's QK^T).  Each
// thread turns 16 bf16 values (two 16-byte loads) into one 16-byte store; the last
// n % 16 elements go one per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const uint4* __restrict__ x,
                                                            uint4* __restrict__ y, long long nvec,
                                                            float scale) {
  const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += step) {
    const uint4 a = x[2 * i], b = x[2 * i + 1];
    y[i] = make_uint4(e4m3x4(a.x, a.y, scale), e4m3x4(a.z, a.w, scale), e4m3x4(b.x, b.y, scale),
                      e4m3x4(b.z, b.w, scale));
  }
}

__global__ void quantize_e4m3_tail_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ y,
                                          int n, float scale) {
  const int i = threadIdx.x;
  if (i < n) {
    const float v = __fmul_rn(__uint_as_float(static_cast<uint32_t>(x[i]) << 16), scale);
    y[i] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
  }
}

cudaError_t launch_quantize_e4m3(const __nv_bfloat16* x, uint8_t* y, long long n, float scale,
                                 cudaStream_t stream) {
  const long long nvec = n / 16;
  if (nvec > 0) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long need = (nvec + 255) / 256;
    const int blocks = static_cast<int>(need < 8LL * sms ? need : 8LL * sms);
    quantize_e4m3_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x),
                                                     reinterpret_cast<uint4*>(y), nvec, scale);
  }
  const int tail = static_cast<int>(n - nvec * 16);
  if (tail > 0)
    quantize_e4m3_tail_kernel<<<1, 32, 0, stream>>>(
        reinterpret_cast<const uint16_t*>(x) + nvec * 16, y + nvec * 16, tail, scale);
  return cudaGetLastError();
}

#ifdef DZ_TEST_HOOKS
__global__ void fill_i32_kernel(int* x, size_t n, int value) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    x[i] = value;
}

cudaError_t launch_fill_i32(int* x, size_t n, int value, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(n / 256 + 1 < 1024 ? n / 256 + 1 : 1024);
  fill_i32_kernel<<<blocks, 256, 0, stream>>>(x, n, value);
  return cudaGetLastError();
}
#endif

}  // namespace dz
