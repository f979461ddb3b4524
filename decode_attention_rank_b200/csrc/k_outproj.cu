// Output through the fused value/output factors on tcgen05 tensor cores
// ("STAR-KV 阅读笔记" section 5.3 and Algorithm 2 steps 7-8):
//     out[b][n] = sum_k y[b][k] * M[k][n],   k = (query head h, value channel j)
// computed swapped, out^T = M^T y^T, so the large operand M^T [D][H*wv] is the
// 128-row A tile (K-major) and the small batch y [rows][H*wv] is the B tile.
//
// The work is HBM-bound on M (268 MB per layer for a LongChat-7B layer with
// r_v = 1024).  Both operands are stored pre-tiled and pre-swizzled, so each
// k-step is two plain bulk copies (16 KB of M and rows*128 B of y) into a ring
// of shared-memory stages.  A persistent grid of one CTA per SM splits the
// (D/128) x (K/64) k-steps evenly (stream-K); a CTA whose range crosses an
// output tile boundary flushes its accumulator there.  Partial sums go to the
// workspace and a small kernel adds them in a fixed order.
#include "tc_common.cuh"

namespace starkv {

int outproj_nb(int rows) { return (std::min(std::max(rows, 1), 256) + 15) / 16 * 16; }

namespace {

constexpr int kOutThreads = 192;  // warp 0 producer, warp 1 MMA, warps 2-5 epilogue

struct OutArgs {
  const uint8_t* M;   // [DT][KT] tiles of 128 x 64 fp16, 16 KB each
  const uint8_t* y;   // [NTILES][KTy] tiles of NB x 64 fp16
  int KTy;            // k-tiles of one row tile of y
  int y_step;         // output tile dt reads y k-tiles dt * y_step .. dt * y_step + KT - 1 (0: all read 0 .. KT - 1)
  float* part;        // [grid.x][slots][NB][128] partial sums
  int NB;             // rows of one B tile (multiple of 16, <= 256)
  int KT, DT;         // k-tiles, output tiles
  int slots;          // partial slots per CTA
  int stages;
  uint32_t tmem_cols;
  uint32_t* status;
};

__device__ __forceinline__ long long unit_begin(int c, int G, long long U) { return (long long)c * U / G; }

__global__ void __launch_bounds__(kOutThreads, 1) k_outproj_tc(OutArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[8], empty[8], seg_done[2], acc_free[2], fin;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x, nt = blockIdx.y;
  const long long U = (long long)a.DT * a.KT;
  const long long u0 = unit_begin(c, G, U), u1 = unit_begin(c + 1, G, U);
  const uint32_t a_bytes = 128 * 128, b_bytes = (uint32_t)a.NB * 128;
  uint8_t* A_s = smem;
  uint8_t* B_s = smem + (size_t)a.stages * a_bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&seg_done[i], 1);
      tc::mbar_init(&acc_free[i], 4);
    }
    tc::mbar_init(&fin, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_base, a.tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // unit u = (output tile u / KT, k-tile u % KT); M tiles are stored in unit order
      int i = 0, s = 0;
      uint32_t ph = 0;
      int kt = (int)(u0 % a.KT);
      const uint8_t* msrc = a.M + (size_t)u0 * a_bytes;
      const uint8_t* ybase = a.y + (size_t)nt * a.KTy * b_bytes;
      int dt = (int)(u0 / a.KT);
      for (long long u = u0; u < u1; ++u, ++i) {
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, a.status)) {
          abort_flag = 1;
          break;
        }
        tc::mbar_expect_tx(&full[s], a_bytes + b_bytes);
        tc::bulk_g2s(A_s + (size_t)s * a_bytes, msrc, a_bytes, &full[s]);
        tc::bulk_g2s(B_s + (size_t)s * b_bytes, ybase + (size_t)(dt * a.y_step + kt) * b_bytes, b_bytes, &full[s]);
        msrc += a_bytes;
        if (++kt == a.KT) {
          kt = 0;
          ++dt;
        }
        if (++s == a.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // copies still in flight land before this CTA may exit
      const int issued = i;
      for (int j = issued - a.stages; j < issued; ++j)
        if (j >= 0) tc::mbar_wait(&full[j % a.stages], (uint32_t)(j / a.stages) & 1u, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16(128, a.NB, false, false, false);
      // descriptors as (low, high) halves, stepped in 16-byte units on the low half
      const uint64_t a0 = tc::sdesc_sw128(tc::smem_u32(A_s), 0, 1024), b0 = tc::sdesc_sw128(tc::smem_u32(B_s), 0, 1024);
      const uint32_t a_lo0 = tc::desc_lo(a0), b_lo0 = tc::desc_lo(b0), d_hi = tc::desc_hi(a0);
      int i = 0, seg = 0, s = 0;
      uint32_t ph = 0;
      int kt = (int)(u0 % a.KT);
      bool first = true;
      for (long long u = u0; u < u1 && !abort_flag; ++u, ++i) {
        const int acc = seg & 1;
        if (first && !tc::mbar_wait(&acc_free[acc], (((uint32_t)seg >> 1) & 1u) ^ 1u, a.status)) {
          abort_flag = 1;
          break;
        }
        if (!tc::mbar_wait(&full[s], ph, a.status)) {
          abort_flag = 1;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * a.NB);
        const uint32_t alo = a_lo0 + (uint32_t)s * (a_bytes >> 4), blo = b_lo0 + (uint32_t)s * (b_bytes >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_f16_ss2(d, alo + 2u * k, d_hi, blo + 2u * k, d_hi, idesc, (first && k == 0) ? 0u : 1u);
        tc::mma_commit(&empty[s]);
        first = false;
        if (++kt == a.KT) kt = 0;
        if (u + 1 == u1 || kt == 0) {
          tc::mma_commit(&seg_done[acc]);
          ++seg;
          first = true;
        }
        if (++s == a.stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      tc::mma_commit(&fin);
      tc::mbar_wait(&fin, 0, a.status);
    }
  } else {
    // epilogue: warps 2..5 cover TMEM lane quarters (warp % 4)
    const int q = warp & 3;
    const int n_local = q * 32 + lane;
    int seg = 0;
    for (long long u = u0; u < u1; ++seg) {
      const long long seg_end = min(u1, (u / a.KT + 1) * a.KT);
      const int dt = (int)(u / a.KT);
      const int acc = seg & 1;
      const bool ok = tc::mbar_wait(&seg_done[acc], ((uint32_t)seg >> 1) & 1u, a.status);
      tc::tc_fence_after();
      const int slot = dt - (int)(u0 / a.KT);
      float* dst = a.part + (((size_t)c * a.slots + slot) * a.NB) * 128 + n_local;
      for (int b0 = 0; b0 < a.NB; b0 += 16) {
        float v[16];
        if (ok) {
          tc::tmem_ld16_sync(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * a.NB + b0), v);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[(size_t)(b0 + i) * 128] = v[i];
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&acc_free[acc]);
      u = seg_end;
      if (!ok) break;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, a.tmem_cols);
}

// out[row][n] = sum over the CTAs whose k-range touched output tile n / 128.
template <typename TO>
__global__ void k_outproj_reduce(const float* __restrict__ part, int G, int KT, int DT, int slots, int NB, int rows,
                                 int D, TO* __restrict__ out) {
  __shared__ long long seg_off[512];
  const int dt = blockIdx.x, row = blockIdx.y;
  const int nt = row / NB, b = row % NB;
  // The CTAs whose unit ranges [begin(c), begin(c + 1)) meet this output
  // tile's k-range [lo, hi): candidates c_lo, c_lo + 1, ... tested one per
  // thread (offset -1 for a CTA that holds none of it), kept in order of c.
  const long long U = (long long)DT * KT;
  const long long lo = (long long)dt * KT, hi = lo + KT;
  const int c_lo = max(0, (int)((lo * G) / U) - 1);
  const int c_hi = min(G, (int)((hi * G + U - 1) / U) + 1);
  const int nc = min(c_hi - c_lo, 512);
  for (int t = threadIdx.x; t < nc; t += blockDim.x) {
    const int c = c_lo + t;
    const long long b0 = unit_begin(c, G, U), b1 = unit_begin(c + 1, G, U);
    long long off = -1;
    if (b1 > b0 && b1 > lo && b0 < hi) {
      const int slot = dt - (int)(b0 / KT);
      off = ((((long long)nt * G + c) * slots + slot) * NB + b) * 128;
    }
    seg_off[t] = off;
  }
  __syncthreads();
  for (int n = threadIdx.x; n < 128; n += blockDim.x) {
    const int d = dt * 128 + n;
    if (d >= D) continue;
    float acc = 0.f;
    for (int k = 0; k < nc; ++k) {
      const long long o = seg_off[k];
      if (o >= 0) acc += part[o + n];
    }
    out[(size_t)row * D + d] = (TO)acc;
  }
}

}  // namespace

// Workspace of the partial sums for `rows` output rows.
// Geometry of a GEMM over an (n_out x K) matrix of 128 x 64 tiles.
OutGeom gemm_geom(int n_out, int K) {
  OutGeom g;
  g.KT = (K + 63) / 64;
  g.DT = (n_out + 127) / 128;
  const long long U = (long long)g.KT * g.DT;
  g.G = (int)std::min<long long>(num_sms(), U);
  const long long per = (U + g.G - 1) / g.G;
  g.slots = (int)((per + g.KT - 1) / g.KT) + 1;
  return g;
}

size_t gemm_part_bytes(int n_out, int K, int rows) {
  const int NB = outproj_nb(rows);
  const int ntiles = (rows + NB - 1) / NB;
  const OutGeom g = gemm_geom(n_out, K);
  return sizeof(float) * (size_t)ntiles * g.G * g.slots * NB * 128;
}

// Unfused output ("STAR-KV 阅读笔记" section 5.3 states the fusion M_h =
// B_v,h W_o,h as an exact reorder, so either order is the same product):
// z_h = y_h B'_v,kv(h) (a grouped GEMM, one 128-output tile per head over that
// head's r_v columns of y), then out = z W_o.  The workspace holds z (fp32),
// z as fp16 B tiles, and the partial sums of either GEMM.
static size_t unfused_z_bytes(const starkv_layer* L, int rows) {
  return ((sizeof(float) * (size_t)rows * L->view.H * L->view.d) + 255) / 256 * 256;
}
static size_t unfused_zt_bytes(const starkv_layer* L, int rows) {
  return (rows_tiles_bytes(rows, L->view.H * L->view.d) + 255) / 256 * 256;
}

size_t outproj_part_bytes(const starkv_layer* L, int rows) {
  if (!L->unfused) return gemm_part_bytes(L->Dp, L->Kp, rows);
  const LayerView& v = L->view;
  return unfused_z_bytes(L, rows) + unfused_zt_bytes(L, rows) +
         std::max(gemm_part_bytes(v.H * v.d, v.wv, rows), gemm_part_bytes(L->Dp, v.H * v.d, rows));
}

cudaError_t launch_gemm_tc(const uint8_t* Mt, int n_out, int K, int n_valid, const void* y_tiles, int rows,
                           void* out, bool out_f32, float* part, uint32_t* status, cudaStream_t s, int y_group) {
  const OutGeom g = gemm_geom(n_out, K);
  const int NB = outproj_nb(rows);
  const int ntiles = (rows + NB - 1) / NB;
  OutArgs a;
  a.M = Mt;
  a.y = (const uint8_t*)y_tiles;
  a.KTy = y_group ? g.KT * g.DT : g.KT;
  a.y_step = y_group ? g.KT : 0;
  a.NB = NB;
  a.KT = g.KT;
  a.DT = g.DT;
  a.slots = g.slots;
  const size_t stage_bytes = 128 * 128 + (size_t)NB * 128;
  a.stages = (int)std::min<size_t>(8, (200 * 1024) / stage_bytes);
  uint32_t cols = 32;
  while (cols < (uint32_t)(2 * NB)) cols <<= 1;
  a.tmem_cols = cols;
  a.status = status;
  const size_t smem = (size_t)a.stages * stage_bytes + 1024;
  cudaError_t e = set_smem_limit((const void*)k_outproj_tc, smem);
  if (e != cudaSuccess) return e;
  for (int t = 0; t < ntiles; ++t) {
    OutArgs at = a;
    at.y = a.y + (size_t)t * a.KTy * NB * 128;
    at.part = part + (size_t)t * g.G * g.slots * NB * 128;
    k_outproj_tc<<<dim3(g.G, 1), kOutThreads, smem, s>>>(at);
  }
  if (out_f32)
    k_outproj_reduce<float><<<dim3(g.DT, rows), 128, 0, s>>>(part, g.G, g.KT, g.DT, g.slots, NB, rows, n_valid,
                                                             (float*)out);
  else
    k_outproj_reduce<__nv_bfloat16><<<dim3(g.DT, rows), 128, 0, s>>>(part, g.G, g.KT, g.DT, g.slots, NB, rows,
                                                                     n_valid, (__nv_bfloat16*)out);
  return cudaGetLastError();
}

cudaError_t launch_outproj_tc(const starkv_layer* L, const void* y_tiles, int rows, void* out, float* part,
                              cudaStream_t s) {
  if (L->unfused) {
    const LayerView& v = L->view;
    uint8_t* w = (uint8_t*)part;
    float* z = (float*)w;
    w += unfused_z_bytes(L, rows);
    void* zt = w;
    w += unfused_zt_bytes(L, rows);
    float* p2 = (float*)w;
    cudaError_t e = launch_gemm_tc((const uint8_t*)L->Bv_tiles, v.H * v.d, v.wv, v.H * v.d, y_tiles, rows, z, true,
                                   p2, L->status, s, 1);
    if (e != cudaSuccess) return e;
    e = launch_pack_rows_tiles_f32(z, rows, v.H * v.d, zt, s);
    if (e != cudaSuccess) return e;
    return launch_gemm_tc((const uint8_t*)L->Wo_tiles, L->Dp, v.H * v.d, v.D, zt, rows, out, false, p2, L->status, s);
  }
  return launch_gemm_tc((const uint8_t*)L->M_T, L->Dp, L->Kp, L->view.D, y_tiles, rows, out,
                        L->view.dtype == STARKV_F32, part, L->status, s);
}

__device__ __forceinline__ float ld_any(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float ld_any(const float* p, size_t i) { return p[i]; }

// fp16 B-operand tiles [rows / NB][K / 64][NB][64] (swizzled, zero padded) from a row-major bf16 or fp32 matrix.
template <typename T>
__global__ void k_pack_rows_tiles(const T* __restrict__ x, int rows, int K, int NB, int KT,
                                  uint8_t* __restrict__ tiles) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // one 8-column chunk
  const int nchunk = KT * 8;
  const int ntiles = (rows + NB - 1) / NB;
  if (idx >= (long long)ntiles * NB * nchunk) return;
  const int row = (int)(idx / nchunk), ch = (int)(idx % nchunk);
  const int kt = ch >> 3, c = ch & 7;
  uint32_t o[4] = {0u, 0u, 0u, 0u};
  if (row < rows) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int k = kt * 64 + c * 8 + i;
      const float f0 = k < K ? ld_any(x, (size_t)row * K + k) : 0.f;
      const float f1 = k + 1 < K ? ld_any(x, (size_t)row * K + k + 1) : 0.f;
      const __half2 h = __floats2half2_rn(f0, f1);
      o[i / 2] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  uint8_t* tile = tiles + ((size_t)(row / NB) * KT + kt) * (size_t)NB * 128;
  *reinterpret_cast<uint4*>(tile + tc::sw128((uint32_t)(row % NB), (uint32_t)c)) = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_pack_rows_tiles(const void* x, int rows, int K, void* tiles, cudaStream_t s, int nb) {
  const int NB = nb > 0 ? nb : outproj_nb(rows);
  const int KT = (K + 63) / 64;
  const int ntiles = (rows + NB - 1) / NB;
  const long long n = (long long)ntiles * NB * KT * 8;
  k_pack_rows_tiles<__nv_bfloat16><<<(unsigned)((n + 255) / 256), 256, 0, s>>>((const __nv_bfloat16*)x, rows, K, NB,
                                                                              KT, (uint8_t*)tiles);
  return cudaGetLastError();
}

cudaError_t launch_pack_rows_tiles_f32(const float* x, int rows, int K, void* tiles, cudaStream_t s, int nb) {
  const int NB = nb > 0 ? nb : outproj_nb(rows);
  const int KT = (K + 63) / 64;
  const int ntiles = (rows + NB - 1) / NB;
  const long long n = (long long)ntiles * NB * KT * 8;
  k_pack_rows_tiles<float><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, rows, K, NB, KT, (uint8_t*)tiles);
  return cudaGetLastError();
}

size_t rows_tiles_bytes(int rows, int K) {
  const int NB = outproj_nb(rows);
  return (size_t)((rows + NB - 1) / NB) * ((K + 63) / 64) * NB * 128;
}

}  // namespace starkv
