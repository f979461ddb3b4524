// Joint-value contraction on tcgen05 tensor cores ("STAR-KV 阅读笔记"
// section 5.3 and Algorithm 2 step 6: stack the heads' probabilities and
// multiply them by the shared low-rank value latent in one matrix product).
//
//     Y_h = sum_t p_h(t) zhat_v(t)       for all query heads h at once
//
// computed transposed, Y^T = Zv^T P^T: the dequantized value latent of a
// 128-token tile is the A operand (M = 128 value channels per block, stored
// MN-major as [token][channel] fp16, which is the order the codes are decoded
// in), the stacked probabilities are B (N = heads, K-major), and Y^T for every
// 128-channel block stays in TMEM for a whole run of super-tiles.
//
// P comes from the score kernel as exp2(s - m_g) per 32-token group; a CTA
// rescales it by exp2(m_g - M) with M the maximum over the CTA's run,
// so no accumulator ever needs rescaling.  The CTA writes one partial
// (M, l, Y) per run of one sequence; a combine kernel merges the runs.
//   warp 0      bulk copies of the value latent blocks of each tile's pages
//   warp 1      tcgen05.mma issue, TMEM allocation
//   warps 2-17  P staging (scaled, fp16), dequantization of the 4/3-bit codes
//               into the A tiles (one thread per token and 32-channel group),
//               and the TMEM epilogue of each run
#include <float.h>

#include "tc_common.cuh"

namespace starkv {

namespace {

constexpr int kValWarps = 16;
constexpr int kValThreads = 64 + 32 * kValWarps;   // producer, MMA, 16 staging/dequant/epilogue warps
constexpr int kVSuper = 256;   // tokens per super-tile (matches the score kernel)

struct ValArgs {
  const uint8_t* pool;
  long long n_pages, page_bytes;
  const int32_t* pt;
  int max_pages;
  const int32_t* seq_lens;
  int vblk_off, vblk_bytes;     // value latent block inside a page
  const GroupDesc* vgrp;        // value latent groups (all of 32 channels)
  int rv, H;
  const __half* P;              // [B][H][P_ld]
  long long P_ld;
  const float* m_st;            // [B][H][n_g]: maximum of each 32-token group
  int n_st;
  int n_g;
  long long U;                  // batch * n_st
  int slots;                    // partial slots per CTA
  float* Y;                     // [G][slots][H][rv]
  float* mseg;                  // [G][slots][H]
  float* lseg;
  uint32_t tmem_cols;
  uint32_t* status;
};

__device__ __forceinline__ long long vunit_lo(int c, int G, long long U) { return (long long)c * U / G; }

// Dequantization of 8 codes of one group into four fp16 pairs, in the chunk
// order (c0,c2) (c1,c3) (c4,c6) (c5,c7): each 16-bit lane holds 1024 + u (an
// exact fp16 integer), one exact subtraction of 1024 + 2^(B-1) and one
// correctly rounded multiply by the fp16 scale give (u - 2^(B-1)) * scale.
// The A tile therefore stores, inside every 8-channel chunk, channels
// 0 2 1 3 4 6 5 7; the combine kernel puts them back in order.
__device__ __forceinline__ uint32_t deq2(uint32_t lanes, __half2 sub, __half2 s2) {
  const uint32_t x = lanes | 0x64006400u;
  __half2 h = *reinterpret_cast<const __half2*>(&x);
  h = __hmul2(__hsub2(h, sub), s2);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 deq8_b4(uint32_t run, __half2 sub, __half2 s2) {
  const uint32_t x01 = __byte_perm(run, 0u, 0x4140u);   // bytes c1c0 | c3c2 into the two 16-bit lanes
  const uint32_t x23 = __byte_perm(run, 0u, 0x4342u);
  uint4 o;
  o.x = deq2(x01 & 0x000F000Fu, sub, s2);           // (c0, c2)
  o.y = deq2((x01 >> 4) & 0x000F000Fu, sub, s2);    // (c1, c3)
  o.z = deq2(x23 & 0x000F000Fu, sub, s2);           // (c4, c6)
  o.w = deq2((x23 >> 4) & 0x000F000Fu, sub, s2);    // (c5, c7)
  return o;
}
__device__ __forceinline__ uint4 deq8_b3(uint32_t run, __half2 sub, __half2 s2) {
  uint4 o;
  o.x = deq2((run & 0x7u) | ((run << 10) & 0x70000u), sub, s2);           // c0 bits 0-2, c2 bits 6-8
  o.y = deq2(((run >> 3) & 0x7u) | ((run << 7) & 0x70000u), sub, s2);     // c1 bits 3-5, c3 bits 9-11
  o.z = deq2(((run >> 12) & 0x7u) | ((run >> 2) & 0x70000u), sub, s2);    // c4 bits 12-14, c6 bits 18-20
  o.w = deq2(((run >> 15) & 0x7u) | ((run >> 5) & 0x70000u), sub, s2);    // c5 bits 15-17, c7 bits 21-23
  return o;
}

__global__ void __launch_bounds__(kValThreads, 1) k_values_tc(ValArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t raw_full[2], raw_empty[2], a_full[2], a_empty[2], p_full[2], p_empty[2];
  __shared__ __align__(8) uint64_t seg_done, acc_free, fin;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ float M_s[64], l_s[64];
  __shared__ int2 vg_s[128];     // per 32-channel value group: code width, code block offset
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int raw_stage = (8 * a.vblk_bytes + 1023) / 1024 * 1024;
  uint8_t* R_s = smem;                              // 2 x raw tile (8 value blocks)
  uint8_t* A_s = R_s + 2 * raw_stage;               // 2 x 32 KB A tiles
  uint8_t* P_s = A_s + 2 * 32768;                   // 2 x (H x 128 fp16, K-major swizzled)
  const int p_stage = a.H * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const long long u0 = vunit_lo(c, G, a.U), u1 = vunit_lo(c + 1, G, a.U);
  const int nblk = a.rv / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&raw_full[s], 1);
      tc::mbar_init(&raw_empty[s], kValWarps);
      tc::mbar_init(&a_full[s], kValWarps);
      tc::mbar_init(&a_empty[s], 1);
      tc::mbar_init(&p_full[s], kValWarps);
      tc::mbar_init(&p_empty[s], 1);
    }
    tc::mbar_init(&seg_done, 1);
    tc::mbar_init(&acc_free, kValWarps);
    tc::mbar_init(&fin, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  for (int g = threadIdx.x; g < a.rv / 32; g += blockDim.x) vg_s[g] = make_int2(a.vgrp[g].bits, a.vgrp[g].code_off);
  if (warp == 1) tc::tmem_alloc(&tmem_base, a.tmem_cols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;

  // The work list: units u0..u1-1 -> tiles (two per unit) with tokens < len.
  if (warp == 0) {
    // warp-wide producer: every lane fetches one page id and issues that page's copy
    int nt = 0;
    for (long long u = u0; u < u1; ++u) {
      if (__shfl_sync(0xffffffffu, abort_flag, 0)) break;
      const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
      const int len = min(a.seq_lens[b], a.max_pages * kPage);
      bool stop = false;
      for (int tile = 0; tile < 2; ++tile) {
        const int t0 = st * kVSuper + tile * 128;
        if (t0 >= len) break;
        const int r = nt & 1;
        const int npg = min(8, (len - t0 + kPage - 1) / kPage);
        int page = 0;
        if (lane < npg) {
          page = a.pt[(size_t)b * a.max_pages + t0 / kPage + lane];
          if (page < 0 || page >= a.n_pages) {
            atomicOr(a.status, kBadPage);
            page = 0;
          }
        }
        bool ok = true;
        if (lane == 0) {
          ok = tc::mbar_wait_ab(&raw_empty[r], (((uint32_t)(nt >> 1)) & 1u) ^ 1u, a.status, &abort_flag);
          if (ok) tc::mbar_expect_tx(&raw_full[r], (uint32_t)(npg * a.vblk_bytes));
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          stop = true;
          break;
        }
        if (lane < npg)
          tc::bulk_g2s(R_s + (size_t)r * raw_stage + (size_t)lane * a.vblk_bytes,
                       a.pool + (size_t)page * a.page_bytes + a.vblk_off, (uint32_t)a.vblk_bytes, &raw_full[r]);
        ++nt;
      }
      if (stop) break;
    }
    if (lane == 0)
      for (int j = max(0, nt - 2); j < nt; ++j) tc::mbar_wait(&raw_full[j & 1], ((uint32_t)(j >> 1)) & 1u, a.status);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_f16(128, a.H, false, true, false);
      int nt = 0, na = 0, seg = 0;
      int cur_b = -1;
      bool first = true;
      for (long long u = u0; u < u1 && !abort_flag; ++u) {
        const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
        const int len = min(a.seq_lens[b], a.max_pages * kPage);
        if (st * kVSuper >= len) continue;
        if (b != cur_b) {
          if (cur_b >= 0) {
            tc::mma_commit(&seg_done);
            ++seg;
          }
          cur_b = b;
          first = true;
          if (!tc::mbar_wait_ab(&acc_free, (((uint32_t)seg) & 1u) ^ 1u, a.status, &abort_flag)) break;
          tc::tc_fence_after();
        }
        for (int tile = 0; tile < 2 && !abort_flag; ++tile) {
          const int t0 = st * kVSuper + tile * 128;
          if (t0 >= len) break;
          const int ps = nt & 1;
          if (!tc::mbar_wait_ab(&p_full[ps], ((uint32_t)(nt >> 1)) & 1u, a.status, &abort_flag)) break;
          tc::tc_fence_after();
          const uint32_t pbase = tc::smem_u32(P_s + (size_t)ps * p_stage);
          for (int cb = 0; cb < nblk; ++cb, ++na) {
            const int as = na & 1;
            if (!tc::mbar_wait_ab(&a_full[as], ((uint32_t)(na >> 1)) & 1u, a.status, &abort_flag)) break;
            tc::tc_fence_after();
            const uint32_t abase = tc::smem_u32(A_s + (size_t)as * 32768);
            const uint32_t d = tmem + (uint32_t)(cb * a.H);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // A: MN-major, 64-channel atoms 1024 B apart, 8-token groups 2048 B apart
              const uint64_t ad = tc::sdesc_sw128(abase + (uint32_t)kk * 4096u, 1024, 2048);
              // B: K-major, 64-token atoms of H rows
              const uint64_t bd = tc::sdesc_sw128(pbase + (uint32_t)(kk >> 2) * (uint32_t)(a.H * 128) +
                                                      (uint32_t)(kk & 3) * 32u,
                                                  0, 1024);
              tc::mma_f16_ss(d, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
            }
            tc::mma_commit(&a_empty[as]);
          }
          tc::mma_commit(&p_empty[ps]);
          first = false;
          ++nt;
        }
      }
      if (cur_b >= 0) tc::mma_commit(&seg_done);
      tc::mma_commit(&fin);
      tc::mbar_wait(&fin, 0, a.status);
    }
  } else {
    // ------------------------------------------------ P staging, dequantization, epilogue
    const int e = warp - 2;            // 0..15
    const int tid = threadIdx.x - 64;  // 0..511
    int nt = 0, na = 0, seg = 0, slot = -1;
    int cur_b = -1;
    const long long ub = u0 / a.n_st;
    auto finish_run = [&]() {
      // epilogue of a run: Y^T from TMEM (lanes = value channels), M and l
      const bool ok = tc::mbar_wait_ab(&seg_done, ((uint32_t)seg) & 1u, a.status, &abort_flag);
      tc::tc_fence_after();
      const int q = warp & 3;
      const size_t base = ((size_t)c * a.slots + slot) * a.H;
      for (int cb = e >> 2; cb < nblk; cb += 4) {
        for (int h0 = 0; h0 < a.H; h0 += 16) {
          float v[16];
          if (ok) {
            tc::tmem_ld16_sync(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cb * a.H + h0), v);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.f;
          }
          const int ch = cb * 128 + q * 32 + lane;     // A-tile position (channel order permuted per 8)
#pragma unroll
          for (int i = 0; i < 16; ++i) a.Y[(base + h0 + i) * a.rv + ch] = v[i];
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&acc_free);
      if (tid < a.H) {
        a.mseg[base + tid] = M_s[tid];
        a.lseg[base + tid] = l_s[tid];
      }
      ++seg;
    };
    // every slot of this CTA starts empty (a run with no valid token leaves l = 0)
    if (tid < a.H)
      for (int sl = 0; sl < a.slots; ++sl) {
        a.mseg[((size_t)c * a.slots + sl) * a.H + tid] = -FLT_MAX;
        a.lseg[((size_t)c * a.slots + sl) * a.H + tid] = 0.f;
      }
    // fixed per-thread roles inside a 128-token tile
    const int tok = tid & 127;            // token of the tile
    const int cq = tid >> 7;              // 32-channel group inside a 128-channel block
    const uint32_t a_off = (uint32_t)(tok >> 3) * 2048u + (uint32_t)(cq >> 1) * 1024u + (uint32_t)(tok & 7) * 128u;
    const uint32_t x7 = (uint32_t)(tok & 7);
    const int ph = tid >> 4, pch = tid & 15;   // P staging: head, 8-token chunk
    for (long long u = u0; u < u1; ++u) {
      const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
      const int len = min(a.seq_lens[b], a.max_pages * kPage);
      if (st * kVSuper >= len) continue;
      if (b != cur_b) {
        if (cur_b >= 0) finish_run();
        cur_b = b;
        slot = (int)(b - ub);
        // run maximum over the CTA's units of this sequence
        asm volatile("bar.sync 1, 512;" ::: "memory");
        if (tid < a.H) {
          float m = -FLT_MAX;
          for (long long uu = u; uu < u1 && uu / a.n_st == b; ++uu) {
            const int s2 = (int)(uu % a.n_st);
            if (s2 * kVSuper < len)
              for (int g = 0; g < kVSuper / 32; ++g)
                m = fmaxf(m, a.m_st[((size_t)b * a.H + tid) * a.n_g + s2 * (kVSuper / 32) + g]);
          }
          M_s[tid] = m;
          l_s[tid] = 0.f;
        }
        asm volatile("bar.sync 1, 512;" ::: "memory");
      }
      for (int tile = 0; tile < 2; ++tile) {
        const int t0 = st * kVSuper + tile * 128;
        if (t0 >= len) break;
        // ---- P^T tile: rows = heads, 128 tokens, K-major swizzled, scaled, fp16
        const int ps = nt & 1;
        tc::mbar_wait_ab(&p_empty[ps], (((uint32_t)(nt >> 1)) & 1u) ^ 1u, a.status, &abort_flag);
        uint8_t* pt_s = P_s + (size_t)ps * p_stage;
        if (ph < a.H) {
          const int tp = t0 + pch * 8;
          const float mg = a.m_st[((size_t)b * a.H + ph) * a.n_g + (tp >> 5)];
          const float f = exp2f(mg - M_s[ph]);
          uint4 raw = make_uint4(0, 0, 0, 0);
          if (tp < len) raw = *reinterpret_cast<const uint4*>(a.P + ((size_t)b * a.H + ph) * a.P_ld + tp);
          __half* hv = reinterpret_cast<__half*>(&raw);
          float lsum = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float p = (tp + i < len) ? __half2float(hv[i]) * f : 0.f;
            hv[i] = __float2half_rn(p);
            lsum += __half2float(hv[i]);
          }
          atomicAdd(&l_s[ph], lsum);
          *reinterpret_cast<uint4*>(pt_s + (pch >> 3) * (a.H * 128) + tc::sw128((uint32_t)ph, (uint32_t)(pch & 7))) =
              raw;
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&p_full[ps]);
        // ---- value latent codes -> A tiles, one 128-channel block at a time
        const int r = nt & 1;
        tc::mbar_wait_ab(&raw_full[r], ((uint32_t)(nt >> 1)) & 1u, a.status, &abort_flag);
        const uint8_t* blk = R_s + (size_t)r * raw_stage + (size_t)(tok >> 4) * a.vblk_bytes;
        const int slot16 = tok & 15;
        const bool tvalid = t0 + tok < len;
        for (int cb = 0; cb < nblk; ++cb, ++na) {
          const int as = na & 1;
          const int gi = cb * 4 + cq;
          const int2 vg = vg_s[gi];
          uint32_t w0 = 0, w1 = 0, w2 = 0, w3 = 0;
          float sc = 0.f;
          if (tvalid) {
            sc = __half2float(reinterpret_cast<const __half*>(blk)[gi * kPage + slot16]);
            const uint32_t* cw = reinterpret_cast<const uint32_t*>(blk + vg.y) + slot16 * vg.x;
            if (vg.x == 4) {
              const uint4 v4 = *reinterpret_cast<const uint4*>(cw);
              w0 = v4.x; w1 = v4.y; w2 = v4.z; w3 = v4.w;
            } else {
              w0 = cw[0]; w1 = cw[1]; w2 = cw[2];
            }
          }
          const __half2 s2 = __floats2half2_rn(sc, sc);
          const float offm = 1024.f + (float)(1 << (vg.x - 1));
          const __half2 sub = __floats2half2_rn(offm, offm);
          uint4 o0, o1, o2, o3;
          if (vg.x == 4) {
            o0 = deq8_b4(w0, sub, s2);
            o1 = deq8_b4(w1, sub, s2);
            o2 = deq8_b4(w2, sub, s2);
            o3 = deq8_b4(w3, sub, s2);
          } else {
            o0 = deq8_b3(w0, sub, s2);
            o1 = deq8_b3(__funnelshift_r(w0, w1, 24), sub, s2);
            o2 = deq8_b3(__funnelshift_r(w1, w2, 16), sub, s2);
            o3 = deq8_b3(w2 >> 8, sub, s2);
          }
          if (!tvalid) o0 = o1 = o2 = o3 = make_uint4(0, 0, 0, 0);
          tc::mbar_wait_ab(&a_empty[as], (((uint32_t)(na >> 1)) & 1u) ^ 1u, a.status, &abort_flag);
          uint8_t* at = A_s + (size_t)as * 32768 + a_off;
          const uint32_t c4 = (uint32_t)(cq & 1) * 4u;     // 8-channel chunk index of this group in its atom
          *reinterpret_cast<uint4*>(at + (((c4 + 0u) ^ x7) << 4)) = o0;
          *reinterpret_cast<uint4*>(at + (((c4 + 1u) ^ x7) << 4)) = o1;
          *reinterpret_cast<uint4*>(at + (((c4 + 2u) ^ x7) << 4)) = o2;
          *reinterpret_cast<uint4*>(at + (((c4 + 3u) ^ x7) << 4)) = o3;
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&a_full[as]);
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&raw_empty[r]);
        ++nt;
      }
    }
    if (cur_b >= 0) finish_run();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, a.tmem_cols);
}

// Merge the runs of each sequence: y = sum exp2(M_r - M) Y_r / sum exp2(M_r - M) l_r,
// written as fp16 B-operand tiles of the output kernel.
__global__ void k_values_combine(const float* __restrict__ Y, const float* __restrict__ mseg,
                                 const float* __restrict__ lseg, int G, long long U, int n_st, int slots, int H,
                                 int rv, int NB, int KT, uint8_t* __restrict__ ytiles) {
  // the runs of sequence b: partial slots of the CTAs whose unit ranges meet [b n_st, (b+1) n_st)
  __shared__ int seg_i[256];
  __shared__ float seg_w[256];
  __shared__ int n_seg;
  __shared__ float inv_den;
  const int b = blockIdx.x, h = blockIdx.y;
  if (threadIdx.x == 0) {
    const long long lo = (long long)b * n_st, hi = lo + n_st;
    int c = (int)((lo * G) / U);
    while (c > 0 && vunit_lo(c, G, U) > lo) --c;
    while (vunit_lo(c + 1, G, U) <= lo) ++c;
    int n = 0;
    float m = -FLT_MAX;
    long long b0 = vunit_lo(c, G, U);
    for (; c < G && b0 < hi && n < 256; ++c) {
      const long long b1 = vunit_lo(c + 1, G, U);
      if (b1 > lo && b1 > b0) {
        const int i = (c * slots + (b - (int)(b0 / n_st))) * H + h;
        if (lseg[i] > 0.f) {
          seg_i[n++] = i;
          m = fmaxf(m, mseg[i]);
        }
      }
      b0 = b1;
    }
    float den = 0.f;
    for (int k = 0; k < n; ++k) {
      seg_w[k] = exp2f(mseg[seg_i[k]] - m);
      den += seg_w[k] * lseg[seg_i[k]];
    }
    n_seg = n;
    inv_den = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  const int ns = n_seg;
  const float idn = inv_den;
  const int nt = b / NB, r = b % NB;
  for (int j = threadIdx.x; j < rv; j += blockDim.x) {
    // position of channel j in the value kernel's A tiles: 1 <-> 2 and 5 <-> 6 inside each chunk of 8
    const int jw = j & 7;
    const int jp = (j & ~7) | (jw == 1 ? 2 : jw == 2 ? 1 : jw == 5 ? 6 : jw == 6 ? 5 : jw);
    float acc = 0.f;
    for (int k = 0; k < ns; ++k) acc += seg_w[k] * Y[(size_t)seg_i[k] * rv + jp];
    const uint32_t kk = (uint32_t)(h * rv + j), cidx = kk & 63u;
    uint8_t* tile = ytiles + ((size_t)nt * KT + (kk >> 6)) * (size_t)NB * 128;
    const uint32_t off = tc::sw128((uint32_t)r, cidx >> 3) + (cidx & 7u) * 2u;
    *reinterpret_cast<__half*>(tile + off) = __float2half_rn(acc * idn);
  }
}

}  // namespace

bool plan_values_tc(starkv_layer* L) {
  const LayerView& v = L->view;
  const starkv_layer_config& c = L->cfg;
  if (!L->tc_scores) return false;
  if (v.rv % 128 != 0 || v.H % 16 != 0 || v.H > 64) return false;
  if ((long long)(v.rv / 128) * v.H > 512) return false;
  const LatentDesc& ld = L->lat[v.L - 1];
  if (ld.n_groups * 32 != v.rv) return false;
  for (int g = 0; g < ld.n_groups; ++g) {
    const GroupDesc& gd = L->grp[ld.group0 + g];
    if (gd.n != 32 || (gd.bits != 3 && gd.bits != 4) || gd.start != g * 32) return false;
  }
  (void)c;
  L->vblk_off = ld.block_off;
  // bytes of the value block: scales + code blocks
  size_t bytes = ld.scale_bytes;
  for (int g = 0; g < ld.n_groups; ++g) bytes += (size_t)kPage * 32 * L->grp[ld.group0 + g].bits / 8;
  L->vblk_bytes = (int)bytes;
  const size_t raw_stage = (8 * bytes + 1023) / 1024 * 1024;
  const size_t smem = 2 * raw_stage + 2 * 32768 + 2 * (size_t)v.H * 256 + 1024;
  return smem <= 226 * 1024;
}

size_t values_tc_ws_bytes(const starkv_layer* L, int batch, int max_len) {
  const int n_st = (max_len + kVSuper - 1) / kVSuper;
  const long long U = (long long)batch * n_st;
  const int G = (int)std::min<long long>(num_sms(), U);
  const long long per = (U + G - 1) / G;
  const int slots = (int)((per + n_st - 1) / n_st) + 1;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  const LayerView& v = L->view;
  return r(sizeof(float) * (size_t)G * slots * v.H * v.rv) + 2 * r(sizeof(float) * (size_t)G * slots * v.H);
}

cudaError_t launch_values_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const ScoreOut& so, void* ws,
                             void* ytiles, cudaStream_t s) {
  const LayerView& v = L->view;
  const int max_len = max_pages * kPage;
  const int n_st = (max_len + kVSuper - 1) / kVSuper;
  const long long U = (long long)batch * n_st;
  const int G = (int)std::min<long long>(num_sms(), U);
  const long long per = (U + G - 1) / G;
  const int slots = (int)((per + n_st - 1) / n_st) + 1;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = (uint8_t*)ws;
  ValArgs a;
  a.pool = pool;
  a.n_pages = n_pages;
  a.page_bytes = (long long)L->page_bytes;
  a.pt = pt;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.vblk_off = L->vblk_off;
  a.vblk_bytes = L->vblk_bytes;
  a.vgrp = L->d_grp + L->lat[v.L - 1].group0;
  a.rv = v.rv;
  a.H = v.H;
  a.P = (const __half*)so.P;
  a.P_ld = so.P_ld;
  a.m_st = so.m_st;
  a.n_st = so.n_st;
  a.n_g = so.n_g;
  a.U = U;
  a.slots = slots;
  a.Y = (float*)w;
  w += r(sizeof(float) * (size_t)G * slots * v.H * v.rv);
  a.mseg = (float*)w;
  w += r(sizeof(float) * (size_t)G * slots * v.H);
  a.lseg = (float*)w;
  uint32_t cols = 32;
  while (cols < (uint32_t)((v.rv / 128) * v.H)) cols <<= 1;
  a.tmem_cols = cols;
  a.status = L->status;
  const size_t raw_stage = (8 * (size_t)L->vblk_bytes + 1023) / 1024 * 1024;
  const size_t smem = 2 * raw_stage + 2 * 32768 + 2 * (size_t)v.H * 256 + 1024;
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(k_values_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  k_values_tc<<<G, kValThreads, smem, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int NB = outproj_nb(batch);
  k_values_combine<<<dim3(batch, v.H), 256, 0, s>>>(a.Y, a.mseg, a.lseg, G, U, n_st, slots, v.H, v.rv, NB,
                                                   L->Kp / 64, (uint8_t*)ytiles);
  return cudaGetLastError();
}

}  // namespace starkv

namespace starkv {

// Workspace of the all-tensor-core decode: scores (W'', P, statistics), value
// partials, the fp16 y tiles and the output kernel's partial sums.
size_t decode_tc_ws_bytes(const starkv_layer* L, int batch, int max_len) {
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  const int NB = outproj_nb(batch);
  const size_t ntiles = (batch + NB - 1) / NB;
  const size_t y_bytes = ntiles * (L->Kp / 64) * (size_t)NB * 128;
  return r(scores_tc_ws_bytes(L, batch, max_len)) + r(values_tc_ws_bytes(L, batch, max_len)) + r(y_bytes) +
         r(outproj_part_bytes(L, batch));
}

cudaError_t launch_decode_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                             void* out, void* ws, size_t ws_bytes, cudaStream_t s) {
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  const int max_len = max_pages * kPage;
  if (ws_bytes < decode_tc_ws_bytes(L, batch, max_len)) return cudaErrorInvalidValue;
  uint8_t* w = (uint8_t*)ws;
  uint8_t* w_scores = w;
  w += r(scores_tc_ws_bytes(L, batch, max_len));
  uint8_t* w_values = w;
  w += r(values_tc_ws_bytes(L, batch, max_len));
  const int NB = outproj_nb(batch);
  const size_t ntiles = (batch + NB - 1) / NB;
  const size_t y_bytes = ntiles * (L->Kp / 64) * (size_t)NB * 128;
  uint8_t* ytiles = w;
  w += r(y_bytes);
  float* part = (float*)w;
  ScoreOut so;
  cudaError_t e = launch_scores_tc(L, pool, n_pages, pt, max_pages, batch, seq_lens, q_pos, q, w_scores, &so, nullptr,
                                   0, s);
  if (e != cudaSuccess) return e;
  if (batch % NB != 0 || L->Kp != L->view.H * L->view.wv) {
    e = cudaMemsetAsync(ytiles, 0, y_bytes, s);
    if (e != cudaSuccess) return e;
  }
  e = launch_values_tc(L, pool, n_pages, pt, max_pages, batch, seq_lens, so, w_values, ytiles, s);
  if (e != cudaSuccess) return e;
  return launch_outproj_tc(L, ytiles, batch, out, part, s);
}

}  // namespace starkv
