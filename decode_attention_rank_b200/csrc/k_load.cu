// Load-time folding of a layer's factors (untimed; once per layer).
//  - projection rows A_T[ch][k] = A[k][ch] for every latent channel;
//  - rotated up-projections B' = R^T B, R the block-wise Hadamard of the
//    latent ("STAR-KV 阅读笔记" section 6.1: the rotation is absorbed into the
//    up projection);
//  - value-side output fusion M_h = B'_v,kv(h) W_o,h (section 5.3), stored as
//    M_T [D][H * wv], the operand layout of the output kernel.
#include "tc_common.cuh"

namespace starkv {

// Element index of (row, col < 64) of a 16-bit tile with 128-byte swizzled rows.
__device__ __forceinline__ uint32_t tc_sw128_elem(uint32_t row, uint32_t col) {
  const uint32_t chunk = col >> 3;
  return ((row >> 3) * 1024u + (row & 7u) * 128u + ((chunk ^ (row & 7u)) << 4)) / 2u + (col & 7u);
}

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, size_t i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

template <typename T>
__global__ void k_transpose_into(const T* __restrict__ src, int rows, int cols, T* __restrict__ dst, int dst_row0,
                                 int dst_ld) {
  __shared__ T tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[(size_t)(dst_row0 + c) * dst_ld + r] = tile[threadIdx.x][i];
  }
}

cudaError_t launch_transpose_into(const void* src, int rows, int cols, int dtype, void* dst, int dst_row0,
                                  int dst_ld, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  if (dtype == STARKV_F32)
    k_transpose_into<float><<<grid, block, 0, s>>>((const float*)src, rows, cols, (float*)dst, dst_row0, dst_ld);
  else
    k_transpose_into<__nv_bfloat16><<<grid, block, 0, s>>>((const __nv_bfloat16*)src, rows, cols,
                                                           (__nv_bfloat16*)dst, dst_row0, dst_ld);
  return cudaGetLastError();
}

// out[j][c] = sum_j' R[j][j'] B[j'][c] for the rows j of one latent; R is the
// direct sum over groups of normalised Sylvester blocks (binary decomposition
// of the group length, largest block first), or the identity.
template <typename T>
__global__ void k_rotate_rows(const T* __restrict__ B, int width, int cols, const GroupDesc* __restrict__ grp,
                              int n_groups, int hadamard, float* __restrict__ out) {
  const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (size_t)width * cols) return;
  const int j = (int)(idx / cols), c = (int)(idx % cols);
  if (!hadamard) {
    out[idx] = ld_f(B, idx);
    return;
  }
  int gs = 0, gn = width;
  for (int g = 0; g < n_groups; ++g)
    if (j >= grp[g].start && j < grp[g].start + grp[g].n) {
      gs = grp[g].start;
      gn = grp[g].n;
    }
  const int o = j - gs;
  int bs = 0, rem = gn, p = 1;
  while (rem > 0) {
    p = 1 << (31 - __clz(rem));
    if (o < bs + p) break;
    bs += p;
    rem -= p;
  }
  double acc = 0.0;
  for (int k = 0; k < p; ++k) {
    const int sgn = __popc((o - bs) & k) & 1;
    const double b = ld_f(B, (size_t)(gs + bs + k) * cols + c);
    acc += sgn ? -b : b;
  }
  out[idx] = (float)(acc / sqrt((double)p));
}

cudaError_t launch_rotate_rows(const starkv_layer* L, const void* B, int dtype, int latent, int cols, float* out,
                               cudaStream_t s) {
  const LatentDesc& ld = L->lat[latent];
  const size_t n = (size_t)ld.width * cols;
  const int threads = 256;
  const unsigned blocks = (unsigned)((n + threads - 1) / threads);
  // group table of this latent, relative to the latent's channels
  const GroupDesc* g = L->d_grp + ld.group0;
  if (dtype == STARKV_F32)
    k_rotate_rows<float><<<blocks, threads, 0, s>>>((const float*)B, ld.width, cols, g, ld.n_groups,
                                                    L->view.hadamard, out);
  else
    k_rotate_rows<__nv_bfloat16><<<blocks, threads, 0, s>>>((const __nv_bfloat16*)B, ld.width, cols, g,
                                                            ld.n_groups, L->view.hadamard, out);
  return cudaGetLastError();
}

// M_T[n][h*wv + j] = sum_p Bsrc[j][kv(h)*d + p] * W_o[h*d + p][n], float32
// accumulation; Bsrc = rotated B_v (joint layers) or the identity (plain
// layers, wv = d).  64 x 64 output tiles, 256 threads, 4 x 4 per thread.
// tiled = 0: row-major [D][H*wv] float32.  tiled = 1: fp16 tiles of 128 x 64
// (n, k) elements, 128-byte swizzled, tile (n/128, k/64) at ((n/128)*KT + k/64) * 16 KB.
template <typename T, typename TO>
__global__ void k_fold_M(const float* __restrict__ Bsrc, int bsrc_ld, const T* __restrict__ Wo, int D, int d,
                         int wv, int group_q, int H, int tiled, int KT, TO* __restrict__ MT) {
  __shared__ float As[16][64];
  __shared__ float Ws[16][65];
  const int h = blockIdx.z, kv = h / group_q;
  const int j0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int p0 = 0; p0 < d; p0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int pp = i / 64, jj = i % 64;
      const int j = j0 + jj, p = p0 + pp;
      float a = 0.f;
      if (j < wv && p < d) a = Bsrc ? Bsrc[(size_t)j * bsrc_ld + kv * d + p] : (j == p ? 1.f : 0.f);
      As[pp][jj] = a;
      const int n = n0 + jj;
      Ws[pp][jj] = (p < d && n < D) ? ld_f(Wo, (size_t)(h * d + p) * D + n) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int pp = 0; pp < 16; ++pp)
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] += As[pp][ty * 4 + a] * Ws[pp][tx * 4 + b];
    __syncthreads();
  }
  for (int a = 0; a < 4; ++a)
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + ty * 4 + a, n = n0 + tx * 4 + b;
      if (j < wv && n < D) {
        const size_t k = (size_t)h * wv + j;
        if (!tiled) {
          MT[(size_t)n * H * wv + k] = (TO)acc[a][b];
        } else {
          const size_t tile = ((size_t)(n >> 7) * KT + (k >> 6)) * (128 * 64);
          const uint32_t off = tc_sw128_elem((uint32_t)(n & 127), (uint32_t)(k & 63));
          MT[tile + off] = (TO)acc[a][b];
        }
      }
    }
}

cudaError_t launch_fold_M(const starkv_layer* L, const float* Bv_rot, const void* W_o, cudaStream_t s) {
  const LayerView& v = L->view;
  dim3 grid((v.D + 63) / 64, (v.wv + 63) / 64, v.H);
  const int bld = v.Hkv * v.d;
  if (v.dtype == STARKV_F32)
    k_fold_M<float, float><<<grid, 256, 0, s>>>(Bv_rot, bld, (const float*)W_o, v.D, v.d, v.wv, v.group_q, v.H, 0,
                                                0, (float*)L->M_T);
  else
    k_fold_M<__nv_bfloat16, __half><<<grid, 256, 0, s>>>(Bv_rot, bld, (const __nv_bfloat16*)W_o, v.D, v.d, v.wv,
                                                         v.group_q, v.H, 1, L->Kp / 64, (__half*)L->M_T);
  return cudaGetLastError();
}

// B'_v per query head as the A operand of the grouped output GEMM: tile
// (h, j / 64) holds rows p < d (output z[h d + p]) and columns j (value
// channel), element B'_v[j][kv(h) d + p], fp16, 128-byte swizzled.
__global__ void k_bv_tiles(const float* __restrict__ Bv_rot, int rv, int d, int Hkv, int group_q, int H,
                           __half* __restrict__ tiles) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)H * rv * d) return;
  const int p = (int)(idx % d);
  const long long r = idx / d;
  const int j = (int)(r % rv), h = (int)(r / rv);
  const int kv = h / group_q;
  const int KT = rv / 64;
  const size_t tile = ((size_t)h * KT + (j >> 6)) * (128 * 64);
  tiles[tile + tc_sw128_elem((uint32_t)p, (uint32_t)(j & 63))] = __float2half_rn(Bv_rot[(size_t)j * Hkv * d + kv * d + p]);
}

cudaError_t launch_build_unfused(starkv_layer* L, const float* Bv_rot, const void* W_o, cudaStream_t s) {
  const LayerView& v = L->view;
  const long long n = (long long)v.H * v.rv * v.d;
  k_bv_tiles<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(Bv_rot, v.rv, v.d, v.Hkv, v.group_q, v.H,
                                                         (__half*)L->Bv_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // W_o^T tiles: the fold with the identity in place of B'_v (k = h d + p)
  dim3 grid((v.D + 63) / 64, (v.d + 63) / 64, v.H);
  k_fold_M<__nv_bfloat16, __half><<<grid, 256, 0, s>>>(nullptr, 0, (const __nv_bfloat16*)W_o, v.D, v.d, v.d,
                                                       v.group_q, v.H, 1, v.H * v.d / 64, (__half*)L->Wo_tiles);
  return cudaGetLastError();
}

}  // namespace starkv

namespace starkv {
namespace {

// One CTA of two roles that share the decode kernels' bounded wait: thread 0
// of warp 1 waits on an mbarrier that nothing will complete (no copy is issued
// and nobody arrives), so the wait gives up after limit_ns, sets the timeout
// bit of the status word and raises the CTA's abort flag; warp 0 waits on a
// second such barrier with the abort flag and drains as soon as it sees it,
// the way the other roles of a decode kernel follow an aborting role.  No
// copy, MMA or TMEM allocation is ever in flight.
__global__ void k_wait_timeout_check(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t never, never2;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&never, 1);
    tc::mbar_init(&never2, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 32) {
    if (!tc::mbar_test_wait(&never, 0)) tc::mbar_wait_slow(&never, 0, status, &abort_flag, limit_ns);
  } else if (threadIdx.x == 0) {
    // bounded by its own limit too (four times the other's), in case the flag is never raised
    if (!tc::mbar_test_wait(&never2, 0)) tc::mbar_wait_slow(&never2, 0, nullptr, &abort_flag, 4 * limit_ns);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_check(uint32_t* status, unsigned long long limit_ns, cudaStream_t s) {
  k_wait_timeout_check<<<1, 64, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace starkv
