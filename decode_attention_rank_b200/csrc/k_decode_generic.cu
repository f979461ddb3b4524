// Generic decode/prefill attention over the paged latent cache, on CUDA cores.
//
// It covers every layer shape and storage option (f32/bf16/quantized, RoPE on
// or off, MHA/GQA, plain layers) and serves as the path for shapes the fused
// kernels do not take.  Steps ("STAR-KV 阅读笔记" Algorithm 2):
//   qprep   RoPE(q) * softmax scale * log2(e)
//   scores  per (row, KV head, 64-token tile): read + dequantize the key
//           latents, reconstruct K = Zhat B' on chip, apply RoPE at each
//           slot's position, score every query head of the group (step 4)
//   value   per (row, token split, 128 value channels): exp2(s - m) over the
//           split, stacked-head accumulation Y_h += p_h(t) zhat_v(t) on the
//           shared joint value latent (steps 5-6)
//   combine merge split partials (m, l, Y) -> y = Y / l
//   out     out = sum_h y_h M_h with the fused factors (steps 7-8)
#include <float.h>

#include "starkv_internal.cuh"

namespace starkv {

namespace {

constexpr int kTile = 64;
constexpr int kVBlock = 128;

__device__ __forceinline__ int row_seq_of(const RowInfo& ri, int row) { return ri.row_seq ? ri.row_seq[row] : row; }
__device__ __forceinline__ int row_pos_of(const RowInfo& ri, int row) {
  return ri.row_pos ? ri.row_pos[row] : ri.row_len[row] - 1;
}
// Visible length of a row, clamped to the page table's capacity (flagged when above it).
__device__ __forceinline__ int row_len_of(const RowInfo& ri, int row, int cap, uint32_t* status, bool flag) {
  int len = ri.row_len[row];
  if (len > cap || len < 0) {
    if (flag) atomicOr(status, kBadPos);
    len = len < 0 ? 0 : cap;
  }
  return len;
}


__device__ __forceinline__ double rope_freq(int p, int d, float log2_theta) {
  return exp2(-(2.0 * p / d) * (double)log2_theta);
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, size_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}

// qrot[row][h][p] = RoPE(q, pos)[p] * scale * log2(e)
template <typename T>
__global__ void k_qprep(LayerView v, const T* __restrict__ q, RowInfo ri, float* __restrict__ qrot) {
  const int row = blockIdx.x, h = blockIdx.y, d = v.d, half = d / 2;
  const T* qh = q + ((size_t)row * v.H + h) * d;
  float* o = qrot + ((size_t)row * v.H + h) * d;
  const int pos = row_pos_of(ri, row);
  for (int p = threadIdx.x; p < half; p += blockDim.x) {
    float a = ldf(qh, p), b = ldf(qh, p + half);
    if (v.rope) {
      double sn, cs;
      sincos((double)pos * rope_freq(p, d, v.rope_log2_theta), &sn, &cs);
      const float a2 = (float)(a * cs - b * sn), b2 = (float)(b * cs + a * sn);
      a = a2;
      b = b2;
    }
    o[p] = a * v.scale_log2;
    o[p + half] = b * v.scale_log2;
  }
}

// Scores (log2 units) S[row][h][t] for one KV head and one 64-token tile.
__global__ void k_scores(LayerView v, const uint8_t* __restrict__ pool, long long n_pages,
                         const int32_t* __restrict__ pt, int max_pages, RowInfo ri, const float* __restrict__ Bk,
                         const int* __restrict__ key_off, const float* __restrict__ qrot, float* __restrict__ S,
                         int S_ld) {
  extern __shared__ float smem[];
  const int row = blockIdx.z, g = blockIdx.y, t0 = blockIdx.x * kTile;
  const int len = row_len_of(ri, row, max_pages * kPage, v.status, threadIdx.x == 0 && t0 == 0 && g == 0);
  if (t0 >= len) return;
  const int nt = min(kTile, len - t0);
  const int b = row_seq_of(ri, row);
  const LatentDesc ld = v.lat[g];
  const int r = ld.width, d = v.d, half = d / 2;
  float* zt = smem;                 // [kTile][r]
  float* Kt = zt + kTile * r;       // [kTile][d]
  for (int idx = threadIdx.x; idx < nt * r; idx += blockDim.x) {
    const int t = idx / r, j = idx % r, tok = t0 + t;
    const int page = pt[(size_t)b * max_pages + tok / kPage];
    float val = 0.f;
    if (page >= 0 && page < n_pages)
      val = latent_value(v, pool + (size_t)page * v.page_bytes + ld.block_off, ld, tok % kPage, j);
    else if (j == 0)
      atomicOr(v.status, kBadPage);
    zt[idx] = val;
  }
  __syncthreads();
  if (v.plain) {
    for (int idx = threadIdx.x; idx < nt * d; idx += blockDim.x) Kt[idx] = zt[idx];
  } else {
    const float* B = Bk + (size_t)key_off[g] * d;
    for (int idx = threadIdx.x; idx < nt * d; idx += blockDim.x) {
      const int t = idx / d, p = idx % d;
      float acc = 0.f;
      for (int j = 0; j < r; ++j) acc += zt[t * r + j] * B[(size_t)j * d + p];
      Kt[idx] = acc;
    }
    if (v.rope) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < nt * half; idx += blockDim.x) {
        const int t = idx / half, p = idx % half;
        double sn, cs;
        sincos((double)(t0 + t) * rope_freq(p, d, v.rope_log2_theta), &sn, &cs);
        const float a = Kt[t * d + p], bb = Kt[t * d + p + half];
        Kt[t * d + p] = (float)(a * cs - bb * sn);
        Kt[t * d + p + half] = (float)(bb * cs + a * sn);
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nt * v.group_q; idx += blockDim.x) {
    const int t = idx % nt, k = idx / nt, h = g * v.group_q + k;
    const float* qh = qrot + ((size_t)row * v.H + h) * d;
    float acc = 0.f;
    for (int p = 0; p < d; ++p) acc += qh[p] * Kt[t * d + p];
    S[((size_t)row * v.H + h) * S_ld + t0 + t] = acc;
  }
}

// Value partials for one (row, split, block of value channels).  Joint
// latents: every query head reads every channel (stacked-head contraction on
// the shared latent).  Plain layers: a block lies inside one KV head's d
// channels and serves that head's query group.
__global__ void k_value(LayerView v, const uint8_t* __restrict__ pool, long long n_pages,
                        const int32_t* __restrict__ pt, int max_pages, RowInfo ri, const float* __restrict__ S,
                        int S_ld, int n_splits, int chunk, int vb, float* __restrict__ pY, float* __restrict__ pm,
                        float* __restrict__ pl) {
  __shared__ float m_s[32];
  __shared__ float p_s[32][33];
  __shared__ float red[kVBlock / 32];
  const int row = blockIdx.z, split = blockIdx.y, cb = blockIdx.x;
  const int len = row_len_of(ri, row, max_pages * kPage, v.status, false);
  const int ts = split * chunk, te = min(len, ts + chunk);
  const int b = row_seq_of(ri, row);
  const LatentDesc ld = v.lat[v.L - 1];
  const int c0 = cb * vb;
  const int c = c0 + threadIdx.x;
  const bool cvalid = threadIdx.x < vb && c < ld.width;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nh = v.plain ? v.group_q : v.H;
  const int hbase = v.plain ? (c0 / v.d) * v.group_q : 0;
  const int jcol = v.plain ? c - (c0 / v.d) * v.d : c;
  const bool first_block = v.plain ? (c0 % v.d == 0) : (cb == 0);
  for (int h0 = 0; h0 < nh; h0 += 32) {
    const int nhc = min(32, nh - h0);
    float acc[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) acc[k] = 0.f;
    float lsum = 0.f;
    for (int k = 0; k < nhc; ++k) {
      const int h = hbase + h0 + k;
      float m = -FLT_MAX;
      for (int t = ts + threadIdx.x; t < te; t += blockDim.x) m = fmaxf(m, S[((size_t)row * v.H + h) * S_ld + t]);
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) red[wid] = m;
      __syncthreads();
      if (threadIdx.x == 0) {
        float mm = red[0];
        for (int w = 1; w < (int)(blockDim.x / 32); ++w) mm = fmaxf(mm, red[w]);
        m_s[k] = mm;
      }
      __syncthreads();
    }
    for (int tt = ts; tt < te; tt += 32) {
      const int ntk = min(32, te - tt);
      for (int idx = threadIdx.x; idx < 32 * nhc; idx += blockDim.x) {
        const int t = idx % 32, k = idx / 32;
        float p = 0.f;
        if (t < ntk) p = exp2f(S[((size_t)row * v.H + hbase + h0 + k) * S_ld + tt + t] - m_s[k]);
        p_s[t][k] = p;
      }
      __syncthreads();
      if (threadIdx.x < nhc)
        for (int t = 0; t < ntk; ++t) lsum += p_s[t][threadIdx.x];
      if (cvalid) {
        for (int t = 0; t < ntk; ++t) {
          const int tok = tt + t;
          const int page = pt[(size_t)b * max_pages + tok / kPage];
          float z = 0.f;
          if (page >= 0 && page < n_pages)
            z = latent_value(v, pool + (size_t)page * v.page_bytes + ld.block_off, ld, tok % kPage, c);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k < nhc) acc[k] += p_s[t][k] * z;
        }
      }
      __syncthreads();
    }
    const size_t base = ((size_t)row * n_splits + split) * v.H;
    if (cvalid)
      for (int k = 0; k < nhc; ++k) pY[(base + hbase + h0 + k) * v.wv + jcol] = acc[k];
    if (first_block && threadIdx.x < nhc) {
      pm[base + hbase + h0 + threadIdx.x] = ts < te ? m_s[threadIdx.x] : -FLT_MAX;
      pl[base + hbase + h0 + threadIdx.x] = lsum;
    }
    __syncthreads();
  }
}

template <typename TY>
__global__ void k_combine(LayerView v, RowInfo ri, int n_splits, const float* __restrict__ pY,
                          const float* __restrict__ pm, const float* __restrict__ pl, TY* __restrict__ y) {
  const int row = blockIdx.x, h = blockIdx.y;
  float m = -FLT_MAX;
  for (int s = 0; s < n_splits; ++s) m = fmaxf(m, pm[((size_t)row * n_splits + s) * v.H + h]);
  float den = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const size_t i = ((size_t)row * n_splits + s) * v.H + h;
    if (pl[i] > 0.f) den += exp2f(pm[i] - m) * pl[i];
  }
  for (int j = threadIdx.x; j < v.wv; j += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const size_t i = ((size_t)row * n_splits + s) * v.H + h;
      if (pl[i] > 0.f) acc += exp2f(pm[i] - m) * pY[i * v.wv + j];
    }
    y[((size_t)row * v.H + h) * v.wv + j] = (TY)(den > 0.f ? acc / den : 0.f);
  }
}

// Same merge, written as fp16 into the swizzled B-operand tiles of the output kernel:
// row r, column k = h*wv + j lives in tile (r / NB, k / 64), row r % NB, column k % 64.
__global__ void k_combine_tiled(LayerView v, int n_splits, const float* __restrict__ pY, const float* __restrict__ pm,
                                const float* __restrict__ pl, int NB, int KT, uint8_t* __restrict__ ytiles) {
  const int row = blockIdx.x, h = blockIdx.y;
  float m = -FLT_MAX;
  for (int s = 0; s < n_splits; ++s) m = fmaxf(m, pm[((size_t)row * n_splits + s) * v.H + h]);
  float den = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const size_t i = ((size_t)row * n_splits + s) * v.H + h;
    if (pl[i] > 0.f) den += exp2f(pm[i] - m) * pl[i];
  }
  const int nt = row / NB, r = row % NB;
  for (int j = threadIdx.x; j < v.wv; j += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const size_t i = ((size_t)row * n_splits + s) * v.H + h;
      if (pl[i] > 0.f) acc += exp2f(pm[i] - m) * pY[i * v.wv + j];
    }
    const uint32_t k = (uint32_t)(h * v.wv + j);
    const uint32_t c = k & 63u;
    uint8_t* tile = ytiles + ((size_t)nt * KT + (k >> 6)) * (size_t)NB * 128;
    const uint32_t off = (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u + (((c >> 3) ^ (uint32_t)(r & 7)) << 4) +
                         (c & 7u) * 2u;
    *reinterpret_cast<__half*>(tile + off) = __float2half_rn(den > 0.f ? acc / den : 0.f);
  }
}

// out[row][n] = sum_k y[row][k] * M_T[n][k]; one warp per output column, eight rows per pass.
template <typename TY, typename TO>
__global__ void k_out(const TY* __restrict__ y, const TY* __restrict__ MT, int rows, int K, int D,
                      TO* __restrict__ out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= D) return;
  const TY* m = MT + (size_t)warp * K;
  for (int r0 = 0; r0 < rows; r0 += 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int k = lane; k < K; k += 32) {
      const float mv = ldf(m, k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (r0 + i < rows) acc[i] += mv * ldf(y, (size_t)(r0 + i) * K + k);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float s = acc[i];
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0 && r0 + i < rows) out[(size_t)(r0 + i) * D + warp] = (TO)s;
    }
  }
}

// Value channels per block: 128 for joint latents; inside one KV head for plain layers.
int value_block(const LayerView& v) { return v.plain ? (v.d <= kVBlock ? v.d : v.d / 2) : kVBlock; }

struct WsPlan {
  size_t qrot, S, pm, pl, pY, y, part, total;
  size_t y_bytes;
  int n_splits, chunk, S_ld;
};

size_t ru256(size_t x) { return (x + 255) / 256 * 256; }

// Token splits: enough (row, split, channel-block) blocks to fill the SMs
// twice over for decode; one split per row for prefill (rows are plenty).
WsPlan plan_ws(const starkv_layer* L, int rows, int max_len, bool prefill) {
  const LayerView& v = L->view;
  WsPlan p{};
  const int cblocks = (v.rv + value_block(v) - 1) / value_block(v);
  int ns = (int)((2 * 148 * 2 + (long long)rows * cblocks - 1) / ((long long)rows * cblocks));
  ns = std::max(1, std::min(ns, (max_len + 511) / 512));
  if (plain_decode_supported(v)) {
    // streaming plain-layer kernel: (row, KV head, split) CTAs, four or more per SM, >= 256 tokens each
    const long long per = (long long)rows * v.Hkv;
    ns = (int)std::max(1LL, std::min((4LL * num_sms() + per - 1) / per, (long long)(max_len + 255) / 256));
  }
  if (prefill) ns = 1;
  p.n_splits = ns;
  p.chunk = (max_len + ns - 1) / ns;
  p.S_ld = max_len;
  const size_t ys = v.dtype == STARKV_F32 ? 4 : 2;
  size_t o = 0;
  p.qrot = o; o += ru256(sizeof(float) * (size_t)rows * v.H * v.d);
  p.S = o;    o += ru256(sizeof(float) * (size_t)rows * v.H * max_len);
  p.pm = o;   o += ru256(sizeof(float) * (size_t)rows * ns * v.H);
  p.pl = o;   o += ru256(sizeof(float) * (size_t)rows * ns * v.H);
  p.pY = o;   o += ru256(sizeof(float) * (size_t)rows * ns * v.H * v.wv);
  if (v.dtype == STARKV_F32) {
    p.y_bytes = ys * (size_t)rows * v.H * v.wv;
    p.y = o;    o += ru256(p.y_bytes);
    p.part = o;
  } else {
    // fp16 tiles [rows / NB][Kp / 64][NB][64] (swizzled) for the tensor-core output kernel
    const int NB = outproj_nb(rows);
    const size_t ntiles = (rows + NB - 1) / NB;
    p.y_bytes = ntiles * (L->Kp / 64) * (size_t)NB * 128;
    p.y = o;    o += ru256(p.y_bytes);
    p.part = o; o += ru256(outproj_part_bytes(L, rows));
  }
  p.total = o;
  return p;
}

}  // namespace

size_t decode_generic_ws_bytes(const starkv_layer* L, int rows, int max_len, bool prefill) {
  return plan_ws(L, rows, max_len, prefill).total;
}

cudaError_t launch_decode_generic(const starkv_layer* L, const uint8_t* pool, long long n_pages,
                                  const int32_t* page_table, int max_pages, int rows, RowInfo ri, int max_len,
                                  const void* q, void* out, void* ws, size_t ws_bytes, bool prefill,
                                  cudaStream_t s, bool tc_scores) {
  const LayerView& v = L->view;
  const WsPlan p = plan_ws(L, rows, max_len, prefill);
  if (ws_bytes < p.total) return cudaErrorInvalidValue;
  char* w = (char*)ws;
  float* qrot = (float*)(w + p.qrot);
  float* S = (float*)(w + p.S);
  float* pm = (float*)(w + p.pm);
  float* pl = (float*)(w + p.pl);
  float* pY = (float*)(w + p.pY);
  void* y = w + p.y;
  if (v.dtype == STARKV_F32)
    k_qprep<float><<<dim3(rows, v.H), 64, 0, s>>>(v, (const float*)q, ri, qrot);
  else
    k_qprep<__nv_bfloat16><<<dim3(rows, v.H), 64, 0, s>>>(v, (const __nv_bfloat16*)q, ri, qrot);
  int rmax = 0;
  for (int g = 0; g < v.Hkv; ++g) rmax = std::max(rmax, L->lat[g].width);
  const size_t smem = sizeof(float) * kTile * (size_t)(rmax + v.d);
  cudaError_t e = set_smem_limit((const void*)k_scores, smem);
  if (e != cudaSuccess) return e;
  if (plain_decode_supported(v) && !tc_scores) {
    // uncompressed bf16 layer: one streaming pass over K and V, partials for the merge below
    e = launch_plain_decode(L, pool, n_pages, page_table, max_pages, rows, ri, qrot, p.n_splits, p.chunk, pY, pm, pl,
                            s);
    if (e != cudaSuccess) return e;
  } else if (tc_scores) {
    // scores (log2 units) from the tensor-core kernel, written into S
    ScoreOut so;
    e = launch_scores_tc(L, pool, n_pages, page_table, max_pages, rows, ri.row_len, ri.row_pos, q, w + p.total, &so,
                         S, p.S_ld, s);
    if (e != cudaSuccess) return e;
  } else {
    k_scores<<<dim3((max_len + kTile - 1) / kTile, v.Hkv, rows), 256, smem, s>>>(
        v, pool, n_pages, page_table, max_pages, ri, L->Bk, L->d_key_off, qrot, S, p.S_ld);
  }
  if (!(plain_decode_supported(v) && !tc_scores)) {
    const int vb = value_block(v);
    const int cblocks = (v.rv + vb - 1) / vb;
    k_value<<<dim3(cblocks, p.n_splits, rows), kVBlock, 0, s>>>(v, pool, n_pages, page_table, max_pages, ri, S,
                                                                p.S_ld, p.n_splits, p.chunk, vb, pY, pm, pl);
  }
  if (v.dtype == STARKV_F32) {
    k_combine<float><<<dim3(rows, v.H), 128, 0, s>>>(v, ri, p.n_splits, pY, pm, pl, (float*)y);
    k_out<float, float><<<(v.D * 32 + 255) / 256, 256, 0, s>>>((const float*)y, (const float*)L->M_T, rows,
                                                                v.H * v.wv, v.D, (float*)out);
    return cudaGetLastError();
  }
  const int NB = outproj_nb(rows);
  const int KT = L->Kp / 64;
  // padding rows and columns of the y tiles must be zero
  if (rows % NB != 0 || L->Kp != v.H * v.wv) {
    e = cudaMemsetAsync(y, 0, p.y_bytes, s);
    if (e != cudaSuccess) return e;
  }
  k_combine_tiled<<<dim3(rows, v.H), 128, 0, s>>>(v, p.n_splits, pY, pm, pl, NB, KT, (uint8_t*)y);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_outproj_tc(L, y, rows, out, (float*)(w + p.part), s);
}

}  // namespace starkv
