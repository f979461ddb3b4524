// Decode attention of an uncompressed (plain) layer on the CUDA cores: the
// protected layers that STAR-KV leaves unfactored ("STAR-KV 阅读笔记",
// Algorithm 1: the first and last layers keep their full K/V), stored as bf16
// K (after RoPE) per KV head and V in the paged cache.
//
// Per query head the step is two matrix-vector products over the cached
// tokens, each 2-byte element feeding one multiply-add per query head of its
// group, far below the tensor cores' ridge: the kernel streams K and V once
// with 16-byte loads and keeps everything else in registers (split-K flash
// decoding: each CTA is one (row, KV head, token split) and writes a partial
// (m, l, Y) that the shared combine kernel merges).
//
// Layout read (see the page format): per page, the K block of KV head g holds
// [slot][d] bf16, the V block [slot][H_kv * d] bf16.  A warp takes whole pages;
// lane l reads the 16-byte chunk l % 16 (eight channels) of slots l / 16 + 2 i,
// i = 0..7, so each load instruction of the warp covers two slots' full rows.
#include <float.h>

#include "starkv_internal.cuh"

namespace starkv {

namespace {

constexpr int kPlainWarps = 4;
constexpr int kPlainMaxGroup = 8;   // query heads per KV head

__device__ __forceinline__ void bf16x8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <int GQ>
__global__ void __launch_bounds__(32 * kPlainWarps) k_plain_decode(LayerView v, const uint8_t* __restrict__ pool,
                                                                   long long n_pages, const int32_t* __restrict__ pt,
                                                                   int max_pages, RowInfo ri,
                                                                   const float* __restrict__ qrot, int n_splits,
                                                                   int chunk, float* __restrict__ pY,
                                                                   float* __restrict__ pm, float* __restrict__ pl) {
  __shared__ float red_m[kPlainWarps][GQ], red_l[kPlainWarps][GQ];
  __shared__ float red_y[kPlainWarps][GQ][128];
  const int split = blockIdx.x, g = blockIdx.y, row = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int len = ri.row_len[row];
  const int cap = max_pages * kPage;
  if (len > cap || len < 0) {
    if (threadIdx.x == 0 && split == 0 && g == 0) atomicOr(v.status, kBadPos);
    len = len < 0 ? 0 : cap;
  }
  const int b = ri.row_seq ? ri.row_seq[row] : row;
  const int ts = split * chunk, te = min(len, ts + chunk);
  const int h0 = g * GQ;
  const int c8 = lane & 15, half = lane >> 4;   // 16-byte chunk of the row, slot parity
  // this lane's eight channels of each query head, already RoPE'd, scaled by softmax scale * log2(e)
  float q[GQ][8];
#pragma unroll
  for (int hh = 0; hh < GQ; ++hh) {
    const float4* qp = reinterpret_cast<const float4*>(qrot + ((size_t)row * v.H + h0 + hh) * 128 + c8 * 8);
    const float4 a = qp[0], bq = qp[1];
    q[hh][0] = a.x; q[hh][1] = a.y; q[hh][2] = a.z; q[hh][3] = a.w;
    q[hh][4] = bq.x; q[hh][5] = bq.y; q[hh][6] = bq.z; q[hh][7] = bq.w;
  }
  float m[GQ], l[GQ], y[GQ][8];
#pragma unroll
  for (int hh = 0; hh < GQ; ++hh) {
    m[hh] = -FLT_MAX;
    l[hh] = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) y[hh][c] = 0.f;
  }
  const LatentDesc kd = v.lat[g], vd = v.lat[v.L - 1];
  const size_t vrow = (size_t)v.rv * 2;   // bytes of one slot's V row (all KV heads)
  const int p0 = ts / kPage, p1 = (te + kPage - 1) / kPage;
  for (int pg = p0 + warp; pg < p1; pg += kPlainWarps) {
    int page = pt[(size_t)b * max_pages + pg];
    if (page < 0 || page >= n_pages) {
      if (lane == 0) atomicOr(v.status, kBadPage);
      page = 0;
    }
    const uint8_t* base = pool + (size_t)page * v.page_bytes;
    const uint8_t* kb = base + kd.block_off + (size_t)half * 256 + c8 * 16;
    const uint8_t* vb = base + vd.block_off + (size_t)half * vrow + (size_t)g * 256 + c8 * 16;
    uint4 kr[8], vr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) kr[i] = *reinterpret_cast<const uint4*>(kb + (size_t)i * 512);
#pragma unroll
    for (int i = 0; i < 8; ++i) vr[i] = *reinterpret_cast<const uint4*>(vb + (size_t)i * 2 * vrow);
    // scores of slots half + 2 i
    float s[GQ][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float kf[8];
      bf16x8(kr[i], kf);
#pragma unroll
      for (int hh = 0; hh < GQ; ++hh) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) a = fmaf(q[hh][c], kf[c], a);
        s[hh][i] = a;
      }
    }
#pragma unroll
    for (int hh = 0; hh < GQ; ++hh)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float a = s[hh][i];
        a += __shfl_xor_sync(0xffffffffu, a, 8);
        a += __shfl_xor_sync(0xffffffffu, a, 4);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        const int t = pg * kPage + half + 2 * i;
        s[hh][i] = (t >= ts && t < te) ? a : -FLT_MAX;
      }
    // online softmax over the page, values
#pragma unroll
    for (int hh = 0; hh < GQ; ++hh) {
      float mx = s[hh][0];
#pragma unroll
      for (int i = 1; i < 8; ++i) mx = fmaxf(mx, s[hh][i]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(m[hh], mx);
      const float alpha = exp2f(m[hh] - mn);
      m[hh] = mn;
      l[hh] *= alpha;
#pragma unroll
      for (int c = 0; c < 8; ++c) y[hh][c] *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float p = s[hh][i] == -FLT_MAX ? 0.f : exp2f(s[hh][i] - mn);
        s[hh][i] = p;
        l[hh] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float vf[8];
      bf16x8(vr[i], vf);
#pragma unroll
      for (int hh = 0; hh < GQ; ++hh)
#pragma unroll
        for (int c = 0; c < 8; ++c) y[hh][c] = fmaf(s[hh][i], vf[c], y[hh][c]);
    }
  }
  // merge the two slot parities of the warp (same channels), then the warps
#pragma unroll
  for (int hh = 0; hh < GQ; ++hh) {
    l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 16);
#pragma unroll
    for (int c = 0; c < 8; ++c) y[hh][c] += __shfl_xor_sync(0xffffffffu, y[hh][c], 16);
    // l: each lane of a 16-lane half summed its own 8 slots' p for every lane of the half; one copy per half
  }
  if (half == 0) {
#pragma unroll
    for (int hh = 0; hh < GQ; ++hh) {
#pragma unroll
      for (int c = 0; c < 8; ++c) red_y[warp][hh][c8 * 8 + c] = y[hh][c];
      if (c8 == 0) {
        red_m[warp][hh] = m[hh];
        red_l[warp][hh] = l[hh];
      }
    }
  }
  __syncthreads();
  // one thread per (head, channel): merge the four warps in a fixed order
  for (int e = threadIdx.x; e < GQ * 128; e += blockDim.x) {
    const int hh = e >> 7, c = e & 127;
    float M = -FLT_MAX;
#pragma unroll
    for (int w = 0; w < kPlainWarps; ++w) M = fmaxf(M, red_m[w][hh]);
    float acc = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kPlainWarps; ++w) {
      const float f = red_l[w][hh] > 0.f ? exp2f(red_m[w][hh] - M) : 0.f;
      acc += f * red_y[w][hh][c];
      den += f * red_l[w][hh];
    }
    const size_t base = ((size_t)row * n_splits + split) * v.H + h0 + hh;
    pY[base * 128 + c] = acc;
    if (c == 0) {
      pm[base] = den > 0.f ? M : -FLT_MAX;
      pl[base] = den;
    }
  }
}

}  // namespace

bool plain_decode_supported(const LayerView& v) {
  return v.plain && v.dtype == STARKV_BF16 && v.d == 128 && v.group_q <= kPlainMaxGroup &&
         (v.group_q & (v.group_q - 1)) == 0;
}

cudaError_t launch_plain_decode(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                                int max_pages, int rows, RowInfo ri, const float* qrot, int n_splits, int chunk,
                                float* pY, float* pm, float* pl, cudaStream_t s) {
  const LayerView& v = L->view;
  const dim3 grid((unsigned)n_splits, (unsigned)v.Hkv, (unsigned)rows);
  switch (v.group_q) {
    case 1: k_plain_decode<1><<<grid, 32 * kPlainWarps, 0, s>>>(v, pool, n_pages, pt, max_pages, ri, qrot, n_splits, chunk, pY, pm, pl); break;
    case 2: k_plain_decode<2><<<grid, 32 * kPlainWarps, 0, s>>>(v, pool, n_pages, pt, max_pages, ri, qrot, n_splits, chunk, pY, pm, pl); break;
    case 4: k_plain_decode<4><<<grid, 32 * kPlainWarps, 0, s>>>(v, pool, n_pages, pt, max_pages, ri, qrot, n_splits, chunk, pY, pm, pl); break;
    case 8: k_plain_decode<8><<<grid, 32 * kPlainWarps, 0, s>>>(v, pool, n_pages, pt, max_pages, ri, qrot, n_splits, chunk, pY, pm, pl); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace starkv
