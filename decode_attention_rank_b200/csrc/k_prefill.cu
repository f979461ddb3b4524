// Causal prefill attention on the tensor cores.
//
// A chunk of new queries of one sequence attends to every cached key up to
// its own position (the causal prefill of a chunked prompt; the model card
// "tenosra/longchat-7b-starkv-proxima" reports a prefill kernel of its own,
// and the pages give no algorithm for it).  Prefill differs from decode in
// that a key is seen by up to a whole chunk of queries, so here the keys and
// values are reconstructed once per chunk, K_h = RoPE(Zhat_k,kv(h) B'_k) and
// V_h = Zhat_v B'_v[:, kv(h)] ("STAR-KV 阅读笔记" section 5.3: keys are
// rebuilt from the pre-RoPE latents and rotated at their positions; the value
// fusion of section 5.3 is an exact reorder, so the output may equally be
// taken through W_o after the values are rebuilt), and the attention itself
// is the standard one over 128 x 128 tiles:
//
//   k_prefill_qrope    cos / sin of the chunk's query positions (shared by all heads)
//   k_prefill_q        Q tiles: RoPE at the query positions, softmax scale * log2(e), fp16
//   k_prefill_zk       the dequantized key latents as fp16 A tiles (r <= 64 channels, zero padded to 64)
//   k_prefill_bkt      B'_k of every KV head as an fp16 B tile (once, at load)
//   k_prefill_zv       the dequantized value latent as fp16 B tiles
//   k_gemm_full        on tcgen05: K = Zhat_k B'_k with RoPE in the epilogue (K tiles); V^T tiles =
//                      (B'_v)^T Zhat_v^T; out = y W_o
//   k_prefill_plain_kv plain layers: their stored K (already rotated) and V as tiles
//   k_flash_prefill    S = Q K^T and O += P V on tcgen05, online softmax in registers
//
// Tiles are 128 rows x 128 fp16 columns stored as two K-major 128-byte
// swizzled atoms of 64 columns (32 KB), the operand layout of the MMAs.
#include <float.h>
#include <math.h>

#include "tc_common.cuh"

namespace starkv {

namespace {

constexpr int kT = 128;            // queries per query tile, keys per key tile
constexpr int kTileB = 32768;      // one 128 x 128 fp16 tile
constexpr int kAtomB = 16384;      // one 128 x 64 atom
constexpr int kMaxPrefillRank = 64;   // key ranks that fit the one 64-channel k-tile of the key rebuild

// Byte offset of element (row, col) inside a tile.
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return (uint32_t)(col >> 6) * kAtomB + tc::sw128((uint32_t)row, (uint32_t)((col & 63) >> 3)) + (uint32_t)(col & 7) * 2u;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------------------ Q tiles
// cos / sin of every (query, pair) of the chunk, shared by all heads: query i
// (position q_start + i), pair p: the angle reduced modulo 2 pi in double,
// then a float sincos.  cs[i][p] = (cos, sin).
__global__ void k_prefill_qrope(float log2_theta, int q_len, int q_start, float2* __restrict__ cs) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= q_len * 64) return;
  const int i = idx >> 6, p = idx & 63;
  const double ang = (double)(q_start + i) * exp2(-(2.0 * p / 128.0) * (double)log2_theta);
  const double two_pi = 6.283185307179586476925286766559;
  float sn, c;
  sincosf((float)(ang - two_pi * rint(ang / two_pi)), &sn, &c);
  cs[idx] = make_float2(c, sn);
}

// Query i of the chunk: RoPE (rotate-half pairs, cos / sin from the table;
// none when the layer has no RoPE), times softmax scale * log2(e), as row
// i % 128 of tile [h][i / 128].  Rows past the chunk are zero.  A thread
// takes (row, 8-pair chunk) items of one head.
__global__ void __launch_bounds__(256) k_prefill_q(LayerView v, const __nv_bfloat16* __restrict__ q, int q_len,
                                                  const float2* __restrict__ cs, int n_qt, uint8_t* __restrict__ Qt) {
  const int qt = blockIdx.x, h = blockIdx.y;
  uint8_t* tile = Qt + ((size_t)h * n_qt + qt) * kTileB;
  for (int e = threadIdx.x; e < kT * 8; e += blockDim.x) {
    const int r = e >> 3, c8 = e & 7;   // row, pairs p = 8 c8 .. 8 c8 + 7 (and p + 64)
    const int i = qt * kT + r;
    const uint4* qr = reinterpret_cast<const uint4*>(q + ((size_t)i * v.H + h) * 128);
    const uint4 ra = i < q_len ? qr[c8] : make_uint4(0, 0, 0, 0);       // elements 8 c8 ..
    const uint4 rb = i < q_len ? qr[8 + c8] : make_uint4(0, 0, 0, 0);   // elements 64 + 8 c8 ..
    const uint32_t aw[4] = {ra.x, ra.y, ra.z, ra.w}, bw[4] = {rb.x, rb.y, rb.z, rb.w};
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float re[2], im[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const float a = __uint_as_float(x ? aw[k] & 0xFFFF0000u : aw[k] << 16);
        const float b = __uint_as_float(x ? bw[k] & 0xFFFF0000u : bw[k] << 16);
        const float2 t = (v.rope && i < q_len) ? cs[(size_t)i * 64 + c8 * 8 + 2 * k + x] : make_float2(1.f, 0.f);
        re[x] = (a * t.x - b * t.y) * v.scale_log2;
        im[x] = (b * t.x + a * t.y) * v.scale_log2;
      }
      lo[k] = pack_half2(re[0], re[1]);
      hi[k] = pack_half2(im[0], im[1]);
    }
    *reinterpret_cast<uint4*>(tile + tile_off(r, c8 * 8)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(tile + tile_off(r, 64 + c8 * 8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
}

// ------------------------------------------------------------------ dequantized key latents (A tiles)
// Tile [g][kt]: 128 tokens x 64 channels (fp16, swizzled); channels past the
// KV head's rank r_g (<= 64) and tokens past T are zero.
__global__ void k_prefill_zk(LayerView v, const uint8_t* __restrict__ pool, long long n_pages,
                             const int32_t* __restrict__ pt_row, int T, int n_kt, int n_kt_l,
                             uint8_t* __restrict__ Zk) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // (g, tile kt, row, chunk)
  if (idx >= (long long)v.Hkv * n_kt * kT * 8) return;
  const int c = (int)(idx & 7);
  const int row = (int)((idx >> 3) % kT);
  const long long gk = (idx >> 3) / kT;
  const int kt = (int)(gk % n_kt), g = (int)(gk / n_kt);
  const int t = kt * kT + row;
  const LatentDesc ld = v.lat[g];
  uint32_t o[4] = {0u, 0u, 0u, 0u};
  if (t < T && c * 8 < ld.width) {
    int page = pt_row[t / kPage];
    if (page < 0 || page >= n_pages) {
      atomicOr(v.status, kBadPage);
      page = 0;
    }
    const uint8_t* blk = pool + (size_t)page * v.page_bytes + ld.block_off;
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const int j = c * 8 + k;
      const float z0 = j < ld.width ? latent_value(v, blk, ld, t % kPage, j) : 0.f;
      const float z1 = j + 1 < ld.width ? latent_value(v, blk, ld, t % kPage, j + 1) : 0.f;
      o[k / 2] = pack_half2(z0, z1);
    }
  }
  uint8_t* tile = Zk + ((size_t)g * n_kt_l + kt) * kAtomB;
  *reinterpret_cast<uint4*>(tile + tc::sw128((uint32_t)row, (uint32_t)c)) = make_uint4(o[0], o[1], o[2], o[3]);
}

// B'_k,g as the B operand of K = Zhat_k B'_k: tile g holds row p (channel of
// K, 0 .. 127), column j (latent channel, 0 .. 63) = B'_k,g[j][p], zero for j >= r_g.
__global__ void k_prefill_bkt(LayerView v, const float* __restrict__ Bk, const int* __restrict__ key_off,
                              uint8_t* __restrict__ Bkt) {
  const int g = blockIdx.x;
  const int r = key_off[g + 1] - key_off[g];
  for (int e = threadIdx.x; e < 128 * 8; e += blockDim.x) {   // (chunk c, row p): consecutive threads, consecutive p
    const int p = e & 127, c = e >> 7;
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const int j = c * 8 + k;
      const float b0 = j < r ? Bk[((size_t)key_off[g] + j) * 128 + p] : 0.f;
      const float b1 = j + 1 < r ? Bk[((size_t)key_off[g] + j + 1) * 128 + p] : 0.f;
      o[k / 2] = pack_half2(b0, b1);
    }
    *reinterpret_cast<uint4*>(Bkt + (size_t)g * kAtomB + tc::sw128((uint32_t)p, (uint32_t)c)) =
        make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ dequantized value latent
// B tiles [kt][rv / 64] of 128 tokens x 64 channels (fp16, swizzled) for the
// V^T product; tokens past T are zero.
__global__ void k_prefill_zv(LayerView v, const uint8_t* __restrict__ pool, long long n_pages,
                             const int32_t* __restrict__ pt_row, int T, int n_kt, uint8_t* __restrict__ Zt) {
  const int KT = v.rv / 64;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // (tile kt, k-tile, row, chunk)
  if (idx >= (long long)n_kt * KT * kT * 8) return;
  const int c = (int)(idx & 7);
  const int row = (int)((idx >> 3) % kT);
  const long long tk = (idx >> 3) / kT;
  const int kk = (int)(tk % KT), kt = (int)(tk / KT);
  const int t = kt * kT + row;
  const LatentDesc ld = v.lat[v.L - 1];
  uint32_t o[4] = {0u, 0u, 0u, 0u};
  if (t < T) {
    int page = pt_row[t / kPage];
    if (page < 0 || page >= n_pages) {
      atomicOr(v.status, kBadPage);
      page = 0;
    }
    const uint8_t* blk = pool + (size_t)page * v.page_bytes + ld.block_off;
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const int j = kk * 64 + c * 8 + k;
      o[k / 2] = pack_half2(latent_value(v, blk, ld, t % kPage, j), latent_value(v, blk, ld, t % kPage, j + 1));
    }
  }
  uint8_t* tile = Zt + ((size_t)kt * KT + kk) * kAtomB;
  *reinterpret_cast<uint4*>(tile + tc::sw128((uint32_t)row, (uint32_t)c)) = make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------ plain layers: stored K, V as tiles
// K block of KV head g: [slot][128] bf16 (already rotated); V block:
// [slot][H_kv 128] bf16.  One CTA per (key tile, KV head); V is transposed
// through shared memory.
__global__ void __launch_bounds__(256) k_prefill_plain_kv(LayerView v, const uint8_t* __restrict__ pool,
                                                         long long n_pages, const int32_t* __restrict__ pt_row,
                                                         int T, int n_kt, uint8_t* __restrict__ Kt,
                                                         uint8_t* __restrict__ Vt) {
  __shared__ __half Vs[kT][kT + 8];
  const int kt = blockIdx.x, g = blockIdx.y;
  const LatentDesc kd = v.lat[g], vd = v.lat[v.L - 1];
  uint8_t* ktile = Kt + ((size_t)g * n_kt + kt) * kTileB;
  uint8_t* vtile = Vt + ((size_t)g * n_kt + kt) * kTileB;
  for (int e = threadIdx.x; e < kT * 16; e += blockDim.x) {   // (token row, 8-channel chunk)
    const int row = e >> 4, c = e & 15;
    const int t = kt * kT + row;
    uint4 kk = make_uint4(0, 0, 0, 0), vv = kk;
    if (t < T) {
      int page = pt_row[t / kPage];
      if (page < 0 || page >= n_pages) {
        atomicOr(v.status, kBadPage);
        page = 0;
      }
      const uint8_t* base = pool + (size_t)page * v.page_bytes;
      kk = *reinterpret_cast<const uint4*>(base + kd.block_off + ((size_t)(t % kPage) * 128 + c * 8) * 2);
      vv = *reinterpret_cast<const uint4*>(base + vd.block_off + ((size_t)(t % kPage) * v.rv + g * 128 + c * 8) * 2);
    }
    const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
    uint32_t ko[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(kw[k] << 16), b = __uint_as_float(kw[k] & 0xFFFF0000u);
      ko[k] = pack_half2(a, b);
      Vs[row][c * 8 + 2 * k] = __float2half_rn(__uint_as_float(vw[k] << 16));
      Vs[row][c * 8 + 2 * k + 1] = __float2half_rn(__uint_as_float(vw[k] & 0xFFFF0000u));
    }
    *reinterpret_cast<uint4*>(ktile + tile_off(row, c * 8)) = make_uint4(ko[0], ko[1], ko[2], ko[3]);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kT * 16; e += blockDim.x) {   // (channel row p, 8-token chunk)
    const int p = e >> 4, c = e & 15;
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2 h = __halves2half2(Vs[c * 8 + 2 * k][p], Vs[c * 8 + 2 * k + 1][p]);
      o[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(vtile + tile_off(p, c * 8)) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ------------------------------------------------------------------ full-K GEMM on tcgen05
// D[m][n] = sum_k A[m][k] B[n][k] for one 128 x 128 output tile, all of K in
// one CTA.  A: 128 x 64 tiles at A + blockIdx.x * a_step_x + blockIdx.y *
// a_step_y, k-tiles 16 KB apart; B likewise.
//   EPI_VT:    the tile is V^T of KV head blockIdx.y, key tile blockIdx.x:
//              written as a flash-attention V^T tile (fp16)
//   EPI_OUT:   out[n][m] for rows n < rows and columns m < n_valid (bf16 or fp32)
//   EPI_KROPE: the tile is K of KV head blockIdx.y, key tile blockIdx.x (rows
//              = tokens, columns = channels): rotated at each token's position
//              with the RoPE table and written as a flash-attention K tile
constexpr int kGemmThreads = 256;
constexpr int kGemmStages = 4;
enum { EPI_VT = 0, EPI_OUT_BF16 = 1, EPI_OUT_F32 = 2, EPI_KROPE = 3 };

struct GemmArgs {
  const uint8_t* A;
  long long a_step_x, a_step_y;
  const uint8_t* B;
  long long b_step_x, b_step_y;
  int KT;
  int stages;           // smem stages of (A, B) k-tiles, <= kGemmStages
  void* out;            // EPI_VT / EPI_KROPE: tiles [blockIdx.y][n_tiles]; EPI_OUT: row-major [rows][ld]
  int n_tiles;
  int rows, n_valid, ld;   // EPI_OUT
  const uint8_t* E;        // EPI_KROPE: RoPE table (null: no rotation)
  uint32_t* status;
};

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm_full(GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages], done;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* Ab = a.A + (size_t)blockIdx.x * a.a_step_x + (size_t)blockIdx.y * a.a_step_y;
  const uint8_t* Bb = a.B + (size_t)blockIdx.x * a.b_step_x + (size_t)blockIdx.y * a.b_step_y;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(&done, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_base, 128);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (warp == 0) {
    if (lane == 0) {
      int k = 0;
      for (; k < a.KT; ++k) {
        const int s = k % a.stages;
        if (!tc::mbar_wait_ab_lazy(&empty[s], (((uint32_t)(k / a.stages)) & 1u) ^ 1u, a.status, &abort_flag)) break;
        tc::mbar_expect_tx(&full[s], 2 * kAtomB);
        tc::bulk_g2s(smem + (size_t)s * 2 * kAtomB, Ab + (size_t)k * kAtomB, kAtomB, &full[s]);
        tc::bulk_g2s(smem + (size_t)s * 2 * kAtomB + kAtomB, Bb + (size_t)k * kAtomB, kAtomB, &full[s]);
      }
      for (int j = max(0, k - a.stages); j < k; ++j)
        tc::mbar_wait(&full[j % a.stages], ((uint32_t)(j / a.stages)) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16(128, 128, false, false, false);
      const uint64_t d0 = tc::sdesc_sw128(tc::smem_u32(smem), 0, 1024);
      const uint32_t lo0 = tc::desc_lo(d0), hi = tc::desc_hi(d0);
      int k = 0;
      for (; k < a.KT && !abort_flag; ++k) {
        const int s = k % a.stages;
        if (!tc::mbar_wait_ab(&full[s], ((uint32_t)(k / a.stages)) & 1u, a.status, &abort_flag)) {
          abort_flag = 1;
          break;
        }
        tc::tc_fence_after();
        const uint32_t alo = lo0 + (uint32_t)(s * 2 * kAtomB >> 4), blo = alo + (uint32_t)(kAtomB >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::mma_f16_ss2(tmem, alo + 2u * kk, hi, blo + 2u * kk, hi, idesc, (k | kk) ? 1u : 0u);
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(&done);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int q = warp & 3;
    const int m = q * 32 + lane;   // TMEM lane = output row m
    const bool ok = tc::mbar_wait_ab(&done, 0, a.status, &abort_flag);
    tc::tc_fence_after();
    if constexpr (EPI == EPI_KROPE) {
      // row m = token blockIdx.x * 128 + m: pairs (p, p + 64) of K rotated at that position
      uint8_t* tile = (uint8_t*)a.out + ((size_t)blockIdx.y * a.n_tiles + blockIdx.x) * kTileB;
      const uint8_t* Et = a.E ? a.E + (size_t)blockIdx.x * kTileB : nullptr;
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float re[16], im[16];
        if (ok) {
          tc::tmem_ld16_sync(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, re);
          tc::tmem_ld16_sync(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(64 + c0), im);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) re[i] = im[i] = 0.f;
        }
        // this row's cos / sin of channels c0 .. c0 + 15: four 16-byte loads of the table row
        uint32_t cw[8], sw[8];
        if (Et) {
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            const uint4 c4 = *reinterpret_cast<const uint4*>(Et + tile_off(m, c0 + 8 * h8));
            const uint4 s4 = *reinterpret_cast<const uint4*>(Et + tile_off(m, 64 + c0 + 8 * h8));
            cw[4 * h8] = c4.x; cw[4 * h8 + 1] = c4.y; cw[4 * h8 + 2] = c4.z; cw[4 * h8 + 3] = c4.w;
            sw[4 * h8] = s4.x; sw[4 * h8 + 1] = s4.y; sw[4 * h8 + 2] = s4.z; sw[4 * h8 + 3] = s4.w;
          }
        } else {
          const __half2 one = __floats2half2_rn(1.f, 1.f), zero = __floats2half2_rn(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            cw[k] = *reinterpret_cast<const uint32_t*>(&one);
            sw[k] = *reinterpret_cast<const uint32_t*>(&zero);
          }
        }
        uint32_t lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float2 cs = __half22float2(*reinterpret_cast<const __half2*>(&cw[i / 2]));
          const float2 sn = __half22float2(*reinterpret_cast<const __half2*>(&sw[i / 2]));
          lo[i / 2] = pack_half2(re[i] * cs.x - im[i] * sn.x, re[i + 1] * cs.y - im[i + 1] * sn.y);
          hi[i / 2] = pack_half2(im[i] * cs.x + re[i] * sn.x, im[i + 1] * cs.y + re[i + 1] * sn.y);
        }
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          *reinterpret_cast<uint4*>(tile + tile_off(m, c0 + h8 * 8)) =
              make_uint4(lo[h8 * 4], lo[h8 * 4 + 1], lo[h8 * 4 + 2], lo[h8 * 4 + 3]);
          *reinterpret_cast<uint4*>(tile + tile_off(m, 64 + c0 + h8 * 8)) =
              make_uint4(hi[h8 * 4], hi[h8 * 4 + 1], hi[h8 * 4 + 2], hi[h8 * 4 + 3]);
        }
      }
    }
    for (int c0 = 0; c0 < (EPI == EPI_KROPE ? 0 : 128); c0 += 16) {
      float x[16];
      if (ok) {
        tc::tmem_ld16_sync(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, x);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
      }
      if constexpr (EPI == EPI_VT) {
        uint8_t* tile = (uint8_t*)a.out + ((size_t)blockIdx.y * a.n_tiles + blockIdx.x) * kTileB;
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8)
          *reinterpret_cast<uint4*>(tile + tile_off(m, c0 + h8 * 8)) =
              make_uint4(pack_half2(x[h8 * 8], x[h8 * 8 + 1]), pack_half2(x[h8 * 8 + 2], x[h8 * 8 + 3]),
                         pack_half2(x[h8 * 8 + 4], x[h8 * 8 + 5]), pack_half2(x[h8 * 8 + 6], x[h8 * 8 + 7]));
      } else {
        const int col = blockIdx.y * 128 + m;
        if (col < a.n_valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int row = blockIdx.x * 128 + c0 + i;
            if (row < a.rows) {
              if constexpr (EPI == EPI_OUT_F32)
                reinterpret_cast<float*>(a.out)[(size_t)row * a.ld + col] = x[i];
              else
                reinterpret_cast<__nv_bfloat16*>(a.out)[(size_t)row * a.ld + col] = __float2bfloat16_rn(x[i]);
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------ flash attention over the tiles
// A persistent grid over (query tile, query head) items.  TMEM: S in two
// 128-column buffers, O in columns 256 .. 383; P(j) (fp16 pairs, 64 columns)
// overwrites the S buffer it came from and is the A operand of O += P V read
// straight from TMEM (the MMAs of the issuing thread run in issue order, so
// S(j + 2) lands in that buffer only after PV(j) has read P(j)).
//   warp 0     bulk copies: each item's Q tile, then its K and V^T tiles into kKV stages
//              (three: the copies run two key tiles ahead of the MMAs)
//   warp 1     MMA issue: S(k + 1) = Q K(k + 1)^T is issued before O += P(k) V(k)
//   warps 4 .. softmax, kSoftWarps per TMEM lane quarter: warp 4 + w + 4 x
//              takes part x (kSoftCols key columns of S, kSoftCols channels
//              of O) of the rows 32 w ..; each thread one query row: S from
//              TMEM, causal mask, the row maximum (the parts exchange theirs
//              through shared memory), P as the fp16 A operand of the next
//              MMA; O is rescaled only when the maximum grew by more than 2^8
//              since the last rescale (P then stays below 256, exact in
//              fp16); at the end y = O / l
constexpr int kSoftWarps = 2;                      // softmax warps per TMEM lane quarter
constexpr int kKV = 3;                             // shared-memory stages of (K, V^T) tiles
constexpr int kSoftCols = 128 / kSoftWarps;        // key columns (and O channels) per softmax warp
constexpr int kFlashThreads = 128 + 128 * kSoftWarps;
constexpr float kRescaleSlack = 8.f;   // log2 units

struct FlashArgs {
  int n_qt_used, H;     // query tiles of this chunk, query heads
  const uint8_t* Q;     // [H][n_qt] tiles
  const uint8_t* K;     // [Hkv][n_kt] tiles: rows = keys, columns = channels
  const uint8_t* Vt;    // [Hkv][n_kt] tiles: rows = channels, columns = keys
  int n_qt, n_kt;
  int q_len, q_start;   // queries at positions q_start .. q_start + q_len - 1
  int group_q;
  float* y;             // [q_len][y_ld]: head h at columns 128 h ..
  int y_ld;
  uint32_t* status;
};

// 2^x (hardware approximation; 2^x for x far below zero flushes to 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]),
      "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]),
      "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

// Work items are (query tile, head) pairs taken longest first: item it is
// query tile n_qt - 1 - it / H (later tiles see more keys), head it % H; CTA c
// takes items c, c + G, ... (a persistent grid, so the causal imbalance is
// spread over all CTAs).  Barrier phases run on across items.
__device__ __forceinline__ int flash_n_kt(const FlashArgs& a, int qt) {
  const int nq = min(kT, a.q_len - qt * kT);
  return (a.q_start + qt * kT + nq - 1) / kT + 1;   // key tiles holding a key visible to the tile
}

// N (16 or 32) consecutive 32-bit TMEM columns of this warp's lane quarter from registers.
template <int N>
__device__ __forceinline__ void tmem_st_p(uint32_t taddr, const uint32_t* v) {
  if constexpr (N == 32) {
    tmem_st32(taddr, reinterpret_cast<const float*>(v));
  } else {
    static_assert(N == 16, "16 or 32 columns");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
  }
}

__global__ void __launch_bounds__(kFlashThreads, 1) k_flash_prefill(FlashArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full, q_empty, kv_full[kKV], kv_empty[kKV], s_full[2], s_free[2], p_full, o_done,
      o_free, fin;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ float xch[kSoftWarps][kT];   // per part and row: the part's row maximum, then its row sum
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* Q_s = smem;
  uint8_t* K_s = Q_s + kTileB;          // kKV stages
  uint8_t* V_s = K_s + kKV * kTileB;    // kKV stages
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.n_qt_used * a.H;
  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    tc::mbar_init(&q_empty, 1);
    for (int s = 0; s < kKV; ++s) {
      tc::mbar_init(&kv_full[s], 1);
      tc::mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&s_full[s], 1);
      tc::mbar_init(&s_free[s], 4 * kSoftWarps);
    }
    tc::mbar_init(&p_full, 4 * kSoftWarps);
    tc::mbar_init(&o_done, 1);
    tc::mbar_init(&o_free, 4 * kSoftWarps);
    tc::mbar_init(&fin, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_base, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t o_col = 256;

  if (warp == 0) {
    // ------------------------------------------------ copies: Q once per item, K and V^T per key tile
    if (lane == 0) {
      int jg = 0, n = 0;   // key tiles and items issued
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++n) {
        const int qt = a.n_qt_used - 1 - it / a.H, h = it % a.H, g = h / a.group_q;
        const int n_kt = flash_n_kt(a, qt);
        if (!(ok = tc::mbar_wait_ab_lazy(&q_empty, ((uint32_t)n & 1u) ^ 1u, a.status, &abort_flag))) break;
        tc::mbar_expect_tx(&q_full, kTileB);
        tc::bulk_g2s(Q_s, a.Q + ((size_t)h * a.n_qt + qt) * kTileB, kTileB, &q_full);
        for (int k = 0; k < n_kt; ++k, ++jg) {
          const int s = jg % kKV;
          if (!(ok = tc::mbar_wait_ab_lazy(&kv_empty[s], (((uint32_t)(jg / kKV)) & 1u) ^ 1u, a.status, &abort_flag)))
            break;
          tc::mbar_expect_tx(&kv_full[s], 2 * kTileB);
          tc::bulk_g2s(K_s + (size_t)s * kTileB, a.K + ((size_t)g * a.n_kt + k) * kTileB, kTileB, &kv_full[s]);
          tc::bulk_g2s(V_s + (size_t)s * kTileB, a.Vt + ((size_t)g * a.n_kt + k) * kTileB, kTileB, &kv_full[s]);
        }
      }
      // let copies in flight land before the CTA can exit
      if (n > 0) tc::mbar_wait(&q_full, ((uint32_t)(n - 1)) & 1u, a.status);
      for (int j = max(0, jg - kKV); j < jg; ++j)
        tc::mbar_wait(&kv_full[j % kKV], ((uint32_t)(j / kKV)) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16(128, 128, false, false, false);
      const uint64_t d0 = tc::sdesc_sw128(tc::smem_u32(smem), 0, 1024);
      const uint32_t base_lo = tc::desc_lo(d0), hi = tc::desc_hi(d0);
      const uint32_t q_lo = base_lo, k_lo = base_lo + (kTileB >> 4), v_lo = base_lo + ((1 + kKV) * kTileB >> 4);
      // S(j) = Q K(j)^T into S buffer j & 1 (j counts key tiles over all items; K in stage j % kKV)
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1, ks = j % kKV;
        if (!tc::mbar_wait_ab(&kv_full[ks], ((uint32_t)(j / kKV)) & 1u, a.status, &abort_flag)) return false;
        if (!tc::mbar_wait_ab(&s_free[s], (((uint32_t)(j >> 1)) & 1u) ^ 1u, a.status, &abort_flag)) return false;
        tc::tc_fence_after();
        const uint32_t kb = k_lo + (uint32_t)(ks * kTileB >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_f16_ss2(tmem + (uint32_t)(s * 128), q_lo + (uint32_t)(kk >> 2) * (kAtomB >> 4) + 2u * (kk & 3), hi,
                          kb + (uint32_t)(kk >> 2) * (kAtomB >> 4) + 2u * (kk & 3), hi, idesc, kk ? 1u : 0u);
        tc::mma_commit(&s_full[s]);
        return true;
      };
      bool ok = true;
      int jg = 0, n = 0;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++n) {
        const int qt = a.n_qt_used - 1 - it / a.H;
        const int n_kt = flash_n_kt(a, qt);
        if (!(ok = tc::mbar_wait_ab(&q_full, (uint32_t)n & 1u, a.status, &abort_flag))) break;
        tc::tc_fence_after();
        if (!(ok = issue_s(jg))) break;
        for (int k = 0; k < n_kt; ++k) {
          if (k + 1 < n_kt && !(ok = issue_s(jg + k + 1))) break;
          if (k + 1 == n_kt) tc::mma_commit(&q_empty);   // every S of this item issued: Q may be replaced
          // O += P(k) V(k); the first of an item overwrites O once the softmax has read the last item's
          if (k == 0 && !(ok = tc::mbar_wait_ab(&o_free, ((uint32_t)n & 1u) ^ 1u, a.status, &abort_flag))) break;
          if (!(ok = tc::mbar_wait_ab(&p_full, (uint32_t)(jg + k) & 1u, a.status, &abort_flag))) break;
          tc::tc_fence_after();
          const int pb = (jg + k) & 1;
          const uint32_t vb = v_lo + (uint32_t)(((jg + k) % kKV) * kTileB >> 4);
          // A = P(j) from TMEM: K = 16 keys per MMA, 8 columns of fp16 pairs
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16_ts(tmem + o_col, tmem + (uint32_t)(pb * 128 + kk * 8),
                           vb + (uint32_t)(kk >> 2) * (kAtomB >> 4) + 2u * (kk & 3), hi, idesc, (k | kk) ? 1u : 0u);
          tc::mma_commit(&o_done);
          tc::mma_commit(&kv_empty[(jg + k) % kKV]);
        }
        jg += n_kt;
      }
      if (!ok) abort_flag = 1;
      // every MMA has completed before the CTA may exit
      tc::mma_commit(&fin);
      tc::mbar_wait(&fin, 0, a.status);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax and output
    const int qq = warp & 3;                      // TMEM lane quarter
    const int x = (warp - 4) >> 2;                // column part
    const int r = qq * 32 + lane;                 // query row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(qq * 32) << 16;
    const int bar_id = 1 + qq;                    // named barrier of the softmax warps of this quarter
    const uint32_t xc = (uint32_t)(kSoftCols * x);   // this warp's first S column / O channel
    bool ok = true;
    int jg = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      const int qt = a.n_qt_used - 1 - it / a.H, h = it % a.H;
      const int q0 = qt * kT;
      const int nq = min(kT, a.q_len - q0);
      const int n_kt = flash_n_kt(a, qt);
      const int pos = a.q_start + q0 + r;         // this row's position
      float m_used = -FLT_MAX, l = 0.f;
      for (int k = 0; k < n_kt; ++k) {
        const int j = jg + k, b = j & 1;
        ok = ok && tc::mbar_wait_ab(&s_full[b], ((uint32_t)(j >> 1)) & 1u, a.status, &abort_flag);
        tc::tc_fence_after();
        float s[kSoftCols];
        if (ok) {
#pragma unroll
          for (int c = 0; c < kSoftCols; c += 32) tmem_ld32(tmem + lane_base + (uint32_t)(b * 128) + xc + c, s + c);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < kSoftCols; ++c) s[c] = 0.f;
        }
        // the S buffer may be overwritten once every warp has it in registers
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s_free[b]);
        // causal mask: key k * 128 + xc + c is visible to the query at `pos` if it is not later
        const int lim = pos - k * kT - (int)xc;   // columns c <= lim are visible
        if (lim < kSoftCols - 1) {
#pragma unroll
          for (int c = 0; c < kSoftCols; ++c)
            if (c > lim) s[c] = -FLT_MAX;
        }
        // maximum in eight independent chains
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
        for (int c = 8; c < kSoftCols; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
        float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        // row maximum over the parts
        xch[x][r] = mx;
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(32 * kSoftWarps) : "memory");
#pragma unroll
        for (int y = 0; y < kSoftWarps; ++y) mx = fmaxf(mx, xch[y][r]);
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(32 * kSoftWarps) : "memory");
        // rescale O only when the maximum moved far enough (both halves decide alike)
        float f = 1.f;
        if (mx > m_used + kRescaleSlack || k == 0) {
          f = k == 0 ? 0.f : ex2_approx(m_used - mx);
          m_used = mx;
        }
        uint32_t p2[kSoftCols / 2];
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // row sum in eight independent chains
#pragma unroll
        for (int c = 0; c < kSoftCols; c += 2) {
          const float e0 = ex2_approx(s[c] - m_used), e1 = ex2_approx(s[c + 1] - m_used);   // masked: 0
          l8[(c >> 1) & 7] += e0 + e1;
          p2[c / 2] = pack_half2(e0, e1);
        }
        const float ls = ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        l = l * f + ls;
        // O is rescaled once the previous PV is done (rare: only when the
        // maximum moved by more than the slack); o_done can then be at most
        // one phase ahead of the one waited for, so skipping waits is safe
        if (k > 0 && f != 1.f) {
          ok = ok && tc::mbar_wait_ab(&o_done, ((uint32_t)(j - 1)) & 1u, a.status, &abort_flag);
          tc::tc_fence_after();
          if (ok) {
#pragma unroll 1
            for (int c = 0; c < kSoftCols; c += 32) {
              float o[32];
              tmem_ld32(tmem + lane_base + o_col + xc + (uint32_t)c, o);
              tc::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= f;
              tmem_st32(tmem + lane_base + o_col + xc + (uint32_t)c, o);
            }
            tc::tmem_st_wait();
          }
        }
        // P into the S buffer's columns for these keys (every part has read its S:
        // the maximum exchange above came after the loads)
        tmem_st_p<kSoftCols / 2>(tmem + lane_base + (uint32_t)(b * 128) + xc / 2, p2);
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&p_full);
      }
      jg += n_kt;
      ok = ok && tc::mbar_wait_ab(&o_done, ((uint32_t)(jg - 1)) & 1u, a.status, &abort_flag);
      tc::tc_fence_after();
      // row sum over the parts
      xch[x][r] = l;
      asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(32 * kSoftWarps) : "memory");
      l = 0.f;
#pragma unroll
      for (int y = 0; y < kSoftWarps; ++y) l += xch[y][r];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool row_ok = r < nq;
#pragma unroll 1
      for (int c = 0; c < kSoftCols; c += 32) {
        float o[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + o_col + xc + (uint32_t)c, o);
          tc::tmem_ld_wait();
        }
        if (row_ok) {
          float* yr = a.y + (size_t)(q0 + r) * a.y_ld + (size_t)h * 128 + xc + c;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(yr + i) =
                ok ? make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv) : make_float4(0, 0, 0, 0);
        }
      }
      // O has been read (and xch is free for the next item)
      tc::tc_fence_before();
      asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(32 * kSoftWarps) : "memory");
      if (lane == 0) tc::mbar_arrive(&o_free);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

struct PrefillWs {
  uint8_t *Qt, *Kt, *Vt, *Zt, *Zk, *yt;
  float* y;
  float2* qcs;   // cos / sin per (query, pair)
};

PrefillWs prefill_ws_layout(const starkv_layer* L, void* ws, int max_T, int max_q) {
  const LayerView& v = L->view;
  const int n_qt = (max_q + kT - 1) / kT, n_kt = (max_T + kT - 1) / kT;
  PrefillWs w;
  uint8_t* p = (uint8_t*)ws;
  w.Qt = p;
  p += al256((size_t)v.H * n_qt * kTileB);
  w.Kt = p;
  p += al256((size_t)v.Hkv * n_kt * kTileB);
  w.Vt = p;
  p += al256((size_t)v.Hkv * n_kt * kTileB);
  w.Zt = p;
  p += al256(v.plain ? 0 : (size_t)n_kt * (v.rv / 64) * kAtomB);
  w.Zk = p;
  p += al256(v.plain ? 0 : (size_t)v.Hkv * n_kt * kAtomB);
  w.y = (float*)p;
  p += al256(sizeof(float) * (size_t)n_qt * kT * v.H * 128);
  w.yt = p;
  p += al256((size_t)n_qt * (v.H * 128 / 64) * kAtomB);
  w.qcs = (float2*)p;
  return w;
}

}  // namespace

// W_o as A tiles [Dp / 128][H d / 64] of 128 x 64 (row n, column k = W_o[k][n]):
// a plain layer's output factors are W_o itself.
static const void* prefill_wo_tiles(const starkv_layer* L) { return L->view.plain ? L->M_T : L->Wo_tiles; }

cudaError_t launch_prefill_bk_tiles(const starkv_layer* L, void* tiles, cudaStream_t s) {
  k_prefill_bkt<<<L->view.Hkv, 256, 0, s>>>(L->view, L->Bk, L->d_key_off, (uint8_t*)tiles);
  return cudaGetLastError();
}

bool prefill_flash_supported(const starkv_layer* L) {
  const LayerView& v = L->view;
  if (v.dtype != STARKV_BF16 || v.d != 128 || !prefill_wo_tiles(L)) return false;
  if (v.plain) return true;
  if (!L->tc_scores || !L->Bv_tiles || !L->Bk_tiles || v.rv % 64 != 0) return false;
  for (int g = 0; g < v.Hkv; ++g)
    if (L->lat[g].width > kMaxPrefillRank) return false;
  return true;
}

size_t prefill_flash_ws_bytes(const starkv_layer* L, int max_T, int max_q) {
  const LayerView& v = L->view;
  const int n_qt = (max_q + kT - 1) / kT, n_kt = (max_T + kT - 1) / kT;
  return al256((size_t)v.H * n_qt * kTileB) + 2 * al256((size_t)v.Hkv * n_kt * kTileB) +
         al256(v.plain ? 0 : (size_t)n_kt * (v.rv / 64) * kAtomB) + al256(v.plain ? 0 : (size_t)v.Hkv * n_kt * kAtomB) +
         al256(sizeof(float) * (size_t)n_qt * kT * v.H * 128) + al256((size_t)n_qt * (v.H * 128 / 64) * kAtomB) +
         al256(sizeof(float2) * (size_t)n_qt * kT * 64);
}

// One chunk of q_len queries of one sequence (page table row pt_row) at
// positions q_start ..; q: [q_len][H][128] bf16; out: [q_len][D] in the layer dtype.
cudaError_t launch_prefill_flash(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt_row,
                                 int q_start, int q_len, const void* q, void* out, void* ws, int max_T, int max_q,
                                 cudaStream_t s) {
  const LayerView& v = L->view;
  const int T = q_start + q_len;
  if (q_len <= 0) return cudaSuccess;
  if (T > max_T || q_len > max_q || (!v.plain && T > L->rope_tiles * 128)) return cudaErrorInvalidValue;
  // tiles this chunk fills, and the strides of the tile arrays (laid out for max_q / max_T)
  const int n_qt = (q_len + kT - 1) / kT, n_kt = (T + kT - 1) / kT;
  const int n_qt_l = (max_q + kT - 1) / kT, n_kt_l = (max_T + kT - 1) / kT;
  PrefillWs w = prefill_ws_layout(L, ws, max_T, max_q);
  cudaError_t e;
  if (v.rope) {
    k_prefill_qrope<<<(q_len * 64 + 255) / 256, 256, 0, s>>>(v.rope_log2_theta, q_len, q_start, w.qcs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  k_prefill_q<<<dim3(n_qt, v.H), 256, 0, s>>>(v, (const __nv_bfloat16*)q, q_len, w.qcs, n_qt_l, w.Qt);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (v.plain) {
    k_prefill_plain_kv<<<dim3(n_kt, v.Hkv), 256, 0, s>>>(v, pool, n_pages, pt_row, T, n_kt_l, w.Kt, w.Vt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    // K = Zhat_k B'_k on the tensor cores, rotated in the epilogue
    const long long nzk = (long long)v.Hkv * n_kt * kT * 8;
    k_prefill_zk<<<(unsigned)((nzk + 255) / 256), 256, 0, s>>>(v, pool, n_pages, pt_row, T, n_kt, n_kt_l, w.Zk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    GemmArgs gk{};
    gk.A = w.Zk;
    gk.a_step_x = kAtomB;
    gk.a_step_y = (long long)n_kt_l * kAtomB;
    gk.B = (const uint8_t*)L->Bk_tiles;
    gk.b_step_y = kAtomB;
    gk.KT = 1;
    gk.stages = 1;
    gk.out = w.Kt;
    gk.n_tiles = n_kt_l;
    gk.E = v.rope ? (const uint8_t*)L->rope_E : nullptr;
    gk.status = v.status;
    const size_t smem1 = 2 * (size_t)kAtomB + 1024;
    if ((e = set_smem_limit((const void*)k_gemm_full<EPI_KROPE>, smem1)) != cudaSuccess) return e;
    k_gemm_full<EPI_KROPE><<<dim3(n_kt, v.Hkv), kGemmThreads, smem1, s>>>(gk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long nz = (long long)n_kt * (v.rv / 64) * kT * 8;
    k_prefill_zv<<<(unsigned)((nz + 255) / 256), 256, 0, s>>>(v, pool, n_pages, pt_row, T, n_kt, w.Zt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // V^T of KV head g = (B'_v columns of g)^T Zhat_v^T: A = the 128 x r_v B'_v tiles of query head g * group_q
    GemmArgs ga{};
    ga.A = (const uint8_t*)L->Bv_tiles;
    ga.a_step_y = (long long)v.group_q * (v.rv / 64) * kAtomB;
    ga.B = w.Zt;
    ga.b_step_x = (long long)(v.rv / 64) * kAtomB;
    ga.KT = v.rv / 64;
    ga.stages = std::min(3, ga.KT);   // three stages: two CTAs per SM overlap one's epilogue with the other's loads
    ga.out = w.Vt;
    ga.n_tiles = n_kt_l;
    ga.status = v.status;
    const size_t smem = (size_t)ga.stages * 2 * kAtomB + 1024;
    if ((e = set_smem_limit((const void*)k_gemm_full<EPI_VT>, smem)) != cudaSuccess) return e;
    k_gemm_full<EPI_VT><<<dim3(n_kt, v.Hkv), kGemmThreads, smem, s>>>(ga);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  FlashArgs fa;
  fa.Q = w.Qt;
  fa.K = w.Kt;
  fa.Vt = w.Vt;
  fa.n_qt = n_qt_l;
  fa.n_kt = n_kt_l;
  fa.n_qt_used = n_qt;
  fa.H = v.H;
  fa.q_len = q_len;
  fa.q_start = q_start;
  fa.group_q = v.group_q;
  fa.y = w.y;
  fa.y_ld = v.H * 128;
  fa.status = v.status;
  const size_t fsmem = (1 + 2 * kKV) * (size_t)kTileB + 1024;
  if ((e = set_smem_limit((const void*)k_flash_prefill, fsmem)) != cudaSuccess) return e;
  k_flash_prefill<<<std::min(num_sms(), n_qt * v.H), kFlashThreads, fsmem, s>>>(fa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // out = y W_o: y as fp16 B tiles of 128 rows, W_o as the A tiles
  if ((e = launch_pack_rows_tiles_f32(w.y, q_len, v.H * 128, w.yt, s, 128)) != cudaSuccess) return e;
  GemmArgs go{};
  go.A = (const uint8_t*)prefill_wo_tiles(L);
  go.a_step_y = (long long)(v.H * 128 / 64) * kAtomB;
  go.B = w.yt;
  go.b_step_x = (long long)(v.H * 128 / 64) * kAtomB;
  go.KT = v.H * 128 / 64;
  go.stages = std::min(3, go.KT);
  go.out = out;
  go.rows = q_len;
  go.n_valid = v.D;
  go.ld = v.D;
  go.status = v.status;
  const size_t smem = (size_t)go.stages * 2 * kAtomB + 1024;
  const void* gk = v.dtype == STARKV_F32 ? (const void*)k_gemm_full<EPI_OUT_F32> : (const void*)k_gemm_full<EPI_OUT_BF16>;
  if ((e = set_smem_limit(gk, smem)) != cudaSuccess) return e;
  const dim3 grid(n_qt, (v.D + 127) / 128);
  if (v.dtype == STARKV_F32)
    k_gemm_full<EPI_OUT_F32><<<grid, kGemmThreads, smem, s>>>(go);
  else
    k_gemm_full<EPI_OUT_BF16><<<grid, kGemmThreads, smem, s>>>(go);
  return cudaGetLastError();
}

}  // namespace starkv
