// Append: latent projection, block-wise Hadamard, quantize and bit-pack into
// the paged cache ("STAR-KV 阅读笔记" Algorithm 2 steps 1-3; section 6.1).
#include "starkv_internal.cuh"

namespace starkv {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// z[i][c] = sum_k x[i][k] * A_T[c][k], float32 accumulation.  One warp per
// latent channel, eight tokens per pass.
template <typename T>
__global__ void k_project(const T* __restrict__ x, const T* __restrict__ AT, int n, int D, int Ltot,
                          float* __restrict__ z) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= Ltot) return;
  const T* a = AT + (size_t)warp * D;
  for (int i0 = 0; i0 < n; i0 += 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int k = lane; k < D; k += 32) {
      const float av = to_f(a[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i0 + i < n) acc[i] += av * to_f(x[(size_t)(i0 + i) * D + k]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = acc[i];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && i0 + i < n) z[(size_t)(i0 + i) * Ltot + warp] = v;
    }
  }
}

cudaError_t launch_project(const starkv_layer* L, const void* x, int n, float* z, cudaStream_t s) {
  const LayerView& v = L->view;
  const int threads = 256;
  const int blocks = (v.Ltot * 32 + threads - 1) / threads;
  if (v.dtype == STARKV_F32)
    k_project<float><<<blocks, threads, 0, s>>>((const float*)x, (const float*)L->A_T, n, v.D, v.Ltot, z);
  else
    k_project<__nv_bfloat16><<<blocks, threads, 0, s>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)L->A_T, n,
                                                        v.D, v.Ltot, z);
  return cudaGetLastError();
}

// Block-wise Hadamard of one group held one channel per lane (lanes >= n hold
// zero): butterflies inside each block of the binary decomposition of n
// (largest block first, so every block starts at a multiple of its size).
__device__ __forceinline__ float group_fwht(float x, int lane, int n) {
  int bs = 0, rem = n, p = 0;
  if (lane < n) {
    while (rem > 0) {
      p = 1 << (31 - __clz(rem));
      if (lane < bs + p) break;
      bs += p;
      rem -= p;
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, m);
    if (m < p) x = (lane & m) ? (y - x) : (x + y);
  }
  if (p > 1) x *= rsqrtf((float)p);
  return x;
}

// One warp per (token, latent).  Quantized latents: per group, amax -> fp32
// scale amax/qmax (IEEE division) -> fp16 rounded up -> codes
// round-half-even(z / scale) clamped to +-qmax, offset by 2^(bits-1), ORed
// into the zeroed page as an LSB-first bitstream at bit (slot*n + i)*bits.
// Unquantized latents are stored in the layer dtype (bf16: round to nearest even).
__global__ void k_pack(LayerView v, uint8_t* __restrict__ pool, long long n_pages, const int32_t* __restrict__ pt,
                       int n_seqs, int max_pages, int n, const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
                       const float* __restrict__ z, int rotate, int rope_keys) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int i = warp / v.L, li = warp % v.L;
  if (i >= n) return;
  const int b = seq_idx[i], t = pos[i];
  if (b < 0 || b >= n_seqs || t < 0 || t >= max_pages * kPage) {
    if (lane == 0) atomicOr(v.status, kBadPos);
    return;
  }
  const int page = pt[(size_t)b * max_pages + t / kPage];
  if (page < 0 || page >= n_pages) {
    if (lane == 0) atomicOr(v.status, kBadPage);
    return;
  }
  const int slot = t % kPage;
  const LatentDesc ld = v.lat[li];
  uint8_t* blk = pool + (size_t)page * v.page_bytes + ld.block_off;
  const float* zi = z + (size_t)i * v.Ltot + ld.ch_off;
  if (!v.quantized) {
    const bool rp = rope_keys && li < v.Hkv;
    const int half = ld.width / 2;
    for (int j = lane; j < ld.width; j += 32) {
      float val = zi[j];
      if (rp) {
        const int p = j < half ? j : j - half;
        const double freq = exp2(-(2.0 * p / ld.width) * (double)v.rope_log2_theta);
        double sn, cs;
        sincos((double)t * freq, &sn, &cs);
        const float a = zi[p], bb = zi[p + half];
        val = j < half ? (float)(a * cs - bb * sn) : (float)(bb * cs + a * sn);
      }
      const size_t o = elem_index(slot, j, ld.width, ld.cmajor);
      if (v.es == 4)
        reinterpret_cast<float*>(blk)[o] = val;
      else
        reinterpret_cast<__nv_bfloat16*>(blk)[o] = __float2bfloat16_rn(val);
    }
    return;
  }
  for (int g = 0; g < ld.n_groups; ++g) {
    const GroupDesc gd = v.grp[ld.group0 + g];
    float x = lane < gd.n ? zi[gd.start + lane] : 0.f;
    if (rotate) x = group_fwht(x, lane, gd.n);
    float amax = lane < gd.n ? fabsf(x) : 0.f;
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int qmax = (1 << (gd.bits - 1)) - 1;
    const float s32 = __fdiv_rn(amax, (float)qmax);
    if (!(s32 <= 65504.f)) {
      if (lane == 0) atomicOr(v.status, kScaleOvf);
      continue;
    }
    const __half s16 = __float2half_ru(s32);
    const float sf = __half2float(s16);
    int q = 0;
    if (sf != 0.f) q = min(max(__float2int_rn(__fdiv_rn(x, sf)), -qmax), qmax);
    const uint32_t u = (uint32_t)(q + (1 << (gd.bits - 1)));
    if (lane == 0) reinterpret_cast<__half*>(blk)[g * kPage + slot] = s16;
    if (lane < gd.n) {
      const uint32_t bit = code_bit(slot, lane, gd.n, gd.bits, ld.cmajor);
      uint32_t* w = reinterpret_cast<uint32_t*>(blk + gd.code_off) + (bit >> 5);
      const uint32_t sh = bit & 31;
      atomicOr(w, u << sh);
      if (sh + gd.bits > 32) atomicOr(w + 1, u >> (32 - sh));
    }
  }
}

// Quantized latents: one warp per (token, group) so that no warp walks a
// latent's groups one after another.
__global__ void k_pack_groups(LayerView v, const int* __restrict__ grp_lat, int n_grp, uint8_t* __restrict__ pool,
                              long long n_pages, const int32_t* __restrict__ pt, int n_seqs, int max_pages, int n,
                              const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
                              const float* __restrict__ z, int rotate) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int i = (int)(warp / n_grp), fg = (int)(warp % n_grp);
  if (i >= n) return;
  const int b = seq_idx[i], t = pos[i];
  const int li = grp_lat[fg];
  const LatentDesc ld = v.lat[li];
  const GroupDesc gd = v.grp[fg];
  const int g = fg - ld.group0;
  const bool first = (g == 0);
  if (b < 0 || b >= n_seqs || t < 0 || t >= max_pages * kPage) {
    if (lane == 0 && first) atomicOr(v.status, kBadPos);
    return;
  }
  const int page = pt[(size_t)b * max_pages + t / kPage];
  if (page < 0 || page >= n_pages) {
    if (lane == 0 && first) atomicOr(v.status, kBadPage);
    return;
  }
  const int slot = t % kPage;
  uint8_t* blk = pool + (size_t)page * v.page_bytes + ld.block_off;
  float x = lane < gd.n ? z[(size_t)i * v.Ltot + ld.ch_off + gd.start + lane] : 0.f;
  if (rotate) x = group_fwht(x, lane, gd.n);
  float amax = lane < gd.n ? fabsf(x) : 0.f;
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int qmax = (1 << (gd.bits - 1)) - 1;
  const float s32 = __fdiv_rn(amax, (float)qmax);
  if (!(s32 <= 65504.f)) {
    if (lane == 0) atomicOr(v.status, kScaleOvf);
    return;
  }
  const __half s16 = __float2half_ru(s32);
  const float sf = __half2float(s16);
  int q = 0;
  if (sf != 0.f) q = min(max(__float2int_rn(__fdiv_rn(x, sf)), -qmax), qmax);
  const uint32_t u = (uint32_t)(q + (1 << (gd.bits - 1)));
  if (lane == 0) reinterpret_cast<__half*>(blk)[g * kPage + slot] = s16;
  if (lane < gd.n) {
    const uint32_t bit = code_bit(slot, lane, gd.n, gd.bits, ld.cmajor);
    uint32_t* w = reinterpret_cast<uint32_t*>(blk + gd.code_off) + (bit >> 5);
    const uint32_t sh = bit & 31;
    atomicOr(w, u << sh);
    if (sh + gd.bits > 32) atomicOr(w + 1, u >> (32 - sh));
  }
}

cudaError_t launch_pack(const starkv_layer* L, uint8_t* pool, long long n_pages, const int32_t* page_table,
                        int n_seqs, int max_pages, int n, const int32_t* seq_idx, const int32_t* positions, const float* z,
                        int rotate, int rope_keys, cudaStream_t s) {
  const LayerView& v = L->view;
  const int threads = 256;
  if (v.quantized && L->d_grp_lat) {
    const int ng = (int)L->grp.size();
    const long long warps = (long long)n * ng;
    k_pack_groups<<<(unsigned)((warps * 32 + threads - 1) / threads), threads, 0, s>>>(
        v, L->d_grp_lat, ng, pool, n_pages, page_table, n_seqs, max_pages, n, seq_idx, positions, z, rotate);
    return cudaGetLastError();
  }
  const long long warps = (long long)n * v.L;
  const unsigned blocks = (unsigned)((warps * 32 + threads - 1) / threads);
  k_pack<<<blocks, threads, 0, s>>>(v, pool, n_pages, page_table, n_seqs, max_pages, n, seq_idx, positions, z, rotate,
                                    rope_keys);
  return cudaGetLastError();
}

}  // namespace starkv
