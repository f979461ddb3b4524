// Key scoring on tcgen05 tensor cores for RoPE'd, head-wise key latents
// ("STAR-KV 阅读笔记" section 5.3 and Algorithm 2 step 4: read and dequantize
// the key latents, reconstruct, apply each position's RoPE and score, without
// writing the reconstructed keys anywhere).
//
// With rotate-half RoPE and K_h = Zhat_h B'_h, the score of token t is
//     s_t = sum_j zhat[t][j] G[t][j],   G = E W''^T,
//     E[t]     = [cos(t theta_p) | sin(t theta_p)]            (t x 128, shared by all heads)
//     W''[j]   = [a_p x_jp + b_p y_jp | b_p x_jp - a_p y_jp]  (r_h x 128, per query)
// where (a_p, b_p) = RoPE(q)(p, p + d/2) * softmax scale * log2(e) and
// (x_jp, y_jp) = B'[j](p, p + d/2).  This is an exact rewrite of
// q' . RoPE_t(zhat B'): G is a 128-deep contraction, so it runs on the
// tensor cores, and the per-token dot with the dequantized latent runs in the
// epilogue straight out of TMEM.
//
// Heads are grouped into MMA items of N <= 128 rows of W'' (an N of 32 per head
// would leave the tensor pipe two-thirds idle); a CTA walks 256-token
// super-tiles (two M = 128 tiles sharing one W'' load) of one sequence.
//   warp 0      bulk copies: RoPE table tiles, W'' item blocks, key latent pages
//   warp 1      tcgen05.mma issue (one thread), TMEM allocation
//   warps 2-17  epilogue (16 warps: TMEM lane quarter x tile x head parity):
//               TMEM -> registers, dequantize + dot, softmax statistics of
//               the super-tile, P = exp2(s - m) as fp16
// Outputs per (sequence, head): P (fp16), and per 32-token group m and l = sum P.
#include <float.h>
#include <math.h>

#include "tc_common.cuh"

namespace starkv {

namespace {

constexpr int kEpiWarps = 16;
constexpr int kScoreThreads = 64 + 32 * kEpiWarps;   // producer, MMA, 16 epilogue warps
constexpr int kSuper = 256;          // tokens per super-tile
constexpr int kETileBytes = 32768;   // one 128-position RoPE tile (128 x 128 fp16)

struct ScoreArgs {
  const uint8_t* pool;
  long long n_pages, page_bytes;
  const int32_t* pt;
  int max_pages;
  const int32_t* seq_lens;
  const uint8_t* E;        // RoPE table tiles
  const uint8_t* W;        // W'' blocks: sequence b at b * w_stride
  long long w_stride;
  const ScoreItem* items;
  int n_items;
  const LatentDesc* lat;
  const GroupDesc* grp;
  int gq;                  // query heads per KV head
  int n_st;                // super-tiles per sequence
  long long U;             // batch * n_st
  __half* P;               // [B][H][P_ld]
  long long P_ld;
  float* m_st;             // [B][H][n_g] per 32-token group
  float* l_st;
  int n_g;
  float* S_dbg;            // optional raw scores [B][H][P_ld]
  int H;
  int w_stage, k_stage, WS, KS;
  uint32_t* status;
};

__device__ __forceinline__ long long unit_lo(int c, int G, long long U) { return (long long)c * U / G; }

// TMEM loads without a wait; tmem_wait() below must follow before any use.
__device__ __forceinline__ void tmem_ld8_nw(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld2_nw(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=f"(v[0]), "=f"(v[1]) : "r"(taddr));
}
// Wait for this thread's TMEM loads; the registers are operands so that no use
// of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait(float* g, float* t) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(g[0]), "+f"(g[1]), "+f"(g[2]), "+f"(g[3]), "+f"(g[4]), "+f"(g[5]), "+f"(g[6]), "+f"(g[7]),
                 "+f"(g[8]), "+f"(g[9]), "+f"(g[10]), "+f"(g[11]), "+f"(g[12]), "+f"(g[13]), "+f"(g[14]),
                 "+f"(g[15]), "+f"(g[16]), "+f"(g[17]), "+f"(g[18]), "+f"(g[19]), "+f"(g[20]), "+f"(g[21]),
                 "+f"(g[22]), "+f"(g[23]), "+f"(g[24]), "+f"(g[25]), "+f"(g[26]), "+f"(g[27]), "+f"(g[28]),
                 "+f"(g[29]), "+f"(g[30]), "+f"(g[31]), "+f"(t[0]), "+f"(t[1]), "+f"(t[2]), "+f"(t[3]),
                 "+f"(t[4]), "+f"(t[5])
               :
               : "memory");
}

// 32 bits of a group's code stream starting at stream bit `bit` (shared memory).
__device__ __forceinline__ uint32_t code_run(const uint8_t* codes, uint32_t bit) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(codes) + (bit >> 5);
  return __funnelshift_r(w[0], w[1], bit & 31u);
}

// Code i of a run, as the float 1 + u / 2^B (u placed in the top mantissa bits).
template <int B, int I>
__device__ __forceinline__ float code_f(uint32_t run) {
  constexpr int sh = 23 - B - I * B;
  const uint32_t x = sh >= 0 ? (run << (sh >= 0 ? sh : 0)) : (run >> (sh < 0 ? -sh : 0));
  return __uint_as_float((x & (((1u << B) - 1u) << (23 - B))) | 0x3F800000u);
}

// acc += sum_i (1 + u_i/2^B) g_i and gs += sum_i g_i over the first `cnt` codes (CNT compile-time bound).
template <int B, int CNT>
__device__ __forceinline__ void dot_run(uint32_t run, const float* g, int cnt, float& acc, float& gs) {
#pragma unroll
  for (int i = 0; i < CNT; ++i) {
    float f;
    switch (i) {
      case 0: f = code_f<B, 0>(run); break;
      case 1: f = code_f<B, 1>(run); break;
      case 2: f = code_f<B, 2>(run); break;
      case 3: f = code_f<B, 3>(run); break;
      case 4: f = code_f<B, 4>(run); break;
      case 5: f = code_f<B, 5>(run); break;
      case 6: f = code_f<B, 6>(run); break;
      default: f = code_f<B, 7>(run); break;
    }
    if (i < cnt) {
      acc = fmaf(f, g[i], acc);
      gs += g[i];
    }
  }
}

// sum over one quantization group of (u - 2^(B-1)) * scale * G for one token:
// nf full 8-code chunks from G[0..32), then `tail` codes from T.
template <int B>
__device__ __forceinline__ float group_dot(const uint8_t* codes, uint32_t bit0, int nf, int tail, const float* G,
                                           const float* T) {
  float acc = 0.f, gs = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (c < nf) dot_run<B, 8>(code_run(codes, bit0 + (uint32_t)(c * 8 * B)), G + 8 * c, 8, acc, gs);
  if (tail) dot_run<B, 6>(code_run(codes, bit0 + (uint32_t)(nf * 8 * B)), T, tail, acc, gs);
  // sum (u - off) g = 2^B sum f g - (2^B + off) sum g
  return (float)(1 << B) * acc - (float)((1 << B) + (1 << (B - 1))) * gs;
}

// Per query head: its key latent's groups (start, n, bits, code offset), the
// latent block's offset inside the item's key range, and its first G column.
struct HeadPlan {
  int ng, blk_rel, hcol, pad;
  int4 grp[4];
};

__global__ void __launch_bounds__(kScoreThreads, 1) k_scores_tc(ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t w_full[4], w_empty[4], k_full[4], k_empty[4], e_full[2], e_empty[2];
  __shared__ __align__(8) uint64_t acc_full[2], acc_free[2], fin;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ ScoreItem items_s[64];
  __shared__ HeadPlan hp_s[64];
  __shared__ float sc_s[4][512];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* E_s = smem;                                   // 2 x 32 KB
  uint8_t* W_s = E_s + 2 * kETileBytes;                  // WS x w_stage
  uint8_t* K_s = W_s + (size_t)a.WS * a.w_stage;         // KS x k_stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const long long u0 = unit_lo(c, G, a.U), u1 = unit_lo(c + 1, G, a.U);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      tc::mbar_init(&w_full[s], 1);
      tc::mbar_init(&w_empty[s], 1);
      tc::mbar_init(&k_full[s], 1);
      tc::mbar_init(&k_empty[s], kEpiWarps);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&e_full[s], 1);
      tc::mbar_init(&e_empty[s], 1);
      tc::mbar_init(&acc_full[s], 1);
      tc::mbar_init(&acc_free[s], kEpiWarps);
    }
    tc::mbar_init(&fin, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  // item table and per-head plans in shared memory
  for (int it = threadIdx.x; it < a.n_items; it += blockDim.x) items_s[it] = a.items[it];
  for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
    HeadPlan hp{};
    const LatentDesc ld = a.lat[h / a.gq];
    int item_key_off = 0, hcol = 0;
    for (int it = 0; it < a.n_items; ++it) {
      const ScoreItem& x = a.items[it];
      if (h >= x.h0 && h < x.h0 + x.nh) {
        item_key_off = x.key_off;
        hcol = x.hcol[h - x.h0];
      }
    }
    hp.ng = min(ld.n_groups, 4);
    hp.blk_rel = ld.block_off - item_key_off;
    hp.hcol = hcol;
    for (int g = 0; g < hp.ng; ++g) {
      const GroupDesc gd = a.grp[ld.group0 + g];
      hp.grp[g] = make_int4(gd.start, gd.n, gd.bits, gd.code_off);
    }
    hp_s[h] = hp;
  }
  if (warp == 1) tc::tmem_alloc(&tmem_base, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int i = 0, uc = 0;
      int nk = 0, nw = 0, ne[2] = {0, 0};   // issued stage fills (for the drain below)
      for (long long u = u0; u < u1 && !abort_flag; ++u) {
        const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
        const int t0 = st * kSuper;
        const int len = min(a.seq_lens[b], a.max_pages * kPage);
        if (t0 >= len) continue;
        const int npg = min(kSuper / kPage, (len - t0 + kPage - 1) / kPage);
        for (int it = 0; it < a.n_items && !abort_flag; ++it, ++i) {
          const ScoreItem item = a.items[it];
          const int ks = i % a.KS, ws = i % a.WS;
          if (!tc::mbar_wait_ab(&k_empty[ks], (((uint32_t)(i / a.KS)) & 1u) ^ 1u, a.status, &abort_flag)) break;
          tc::mbar_expect_tx(&k_full[ks], (uint32_t)(npg * item.key_bytes));
          for (int pg = 0; pg < npg; ++pg) {
            int page = a.pt[(size_t)b * a.max_pages + st * (kSuper / kPage) + pg];
            if (page < 0 || page >= a.n_pages) {
              atomicOr(a.status, kBadPage);
              page = 0;
            }
            tc::bulk_g2s(K_s + (size_t)ks * a.k_stage + (size_t)pg * item.key_bytes,
                         a.pool + (size_t)page * a.page_bytes + item.key_off, (uint32_t)item.key_bytes, &k_full[ks]);
          }
          ++nk;
          if (!tc::mbar_wait_ab(&w_empty[ws], (((uint32_t)(i / a.WS)) & 1u) ^ 1u, a.status, &abort_flag)) break;
          tc::mbar_expect_tx(&w_full[ws], (uint32_t)(item.npad * 256));
          tc::bulk_g2s(W_s + (size_t)ws * a.w_stage, a.W + (size_t)b * a.w_stride + item.w_off,
                       (uint32_t)(item.npad * 256), &w_full[ws]);
          ++nw;
          if (it == 0) {
            for (int k = 0; k < 2; ++k) {
              if (!tc::mbar_wait_ab(&e_empty[k], ((uint32_t)uc & 1u) ^ 1u, a.status, &abort_flag)) break;
              tc::mbar_expect_tx(&e_full[k], kETileBytes);
              tc::bulk_g2s(E_s + k * kETileBytes, a.E + (size_t)(t0 / 128 + k) * kETileBytes, kETileBytes,
                           &e_full[k]);
              ++ne[k];
            }
          }
        }
        ++uc;
      }
      // let copies in flight land before the CTA can exit
      for (int j = max(0, nk - a.KS); j < nk; ++j)
        tc::mbar_wait(&k_full[j % a.KS], ((uint32_t)(j / a.KS)) & 1u, a.status);
      for (int j = max(0, nw - a.WS); j < nw; ++j)
        tc::mbar_wait(&w_full[j % a.WS], ((uint32_t)(j / a.WS)) & 1u, a.status);
      for (int k = 0; k < 2; ++k)
        if (ne[k] > 0) tc::mbar_wait(&e_full[k], (uint32_t)(ne[k] - 1) & 1u, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int i = 0, uc = 0;
      for (long long u = u0; u < u1 && !abort_flag; ++u) {
        const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
        const int len = min(a.seq_lens[b], a.max_pages * kPage);
        if (st * kSuper >= len) continue;
        for (int it = 0; it < a.n_items && !abort_flag; ++it, ++i) {
          const int npad = a.items[it].npad;
          const int ws = i % a.WS;
          if (!tc::mbar_wait_ab(&w_full[ws], ((uint32_t)(i / a.WS)) & 1u, a.status, &abort_flag)) { abort_flag = 1; break; }
          if (it == 0) {
            if (!tc::mbar_wait_ab(&e_full[0], (uint32_t)uc & 1u, a.status, &abort_flag) ||
                !tc::mbar_wait_ab(&e_full[1], (uint32_t)uc & 1u, a.status, &abort_flag)) { abort_flag = 1; break; }
          }
          if (!tc::mbar_wait_ab(&acc_free[i & 1], (((uint32_t)(i >> 1)) & 1u) ^ 1u, a.status, &abort_flag)) { abort_flag = 1; break; }
          tc::tc_fence_after();
          const uint32_t idesc = tc::idesc_f16(128, npad, false, false, false);
          const uint32_t wbase = tc::smem_u32(W_s + (size_t)ws * a.w_stage);
          const uint32_t watom = (uint32_t)npad * 128u;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint32_t ebase = tc::smem_u32(E_s + k * kETileBytes);
            const uint32_t d = tmem + (uint32_t)((i & 1) * 256 + k * 128);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ea = ebase + (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u;
              const uint32_t wa = wbase + (uint32_t)(kk >> 2) * watom + (uint32_t)(kk & 3) * 32u;
              tc::mma_f16_ss(d, tc::sdesc_sw128(ea, 0, 1024), tc::sdesc_sw128(wa, 0, 1024), idesc, kk ? 1u : 0u);
            }
          }
          tc::mma_commit(&w_empty[ws]);
          tc::mma_commit(&acc_full[i & 1]);
          if (it == a.n_items - 1) {
            tc::mma_commit(&e_empty[0]);
            tc::mma_commit(&e_empty[1]);
          }
        }
        ++uc;
      }
      tc::mma_commit(&fin);
      tc::mbar_wait(&fin, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // 16 warps: TMEM lane quarter q = warp % 4, tile k, head parity hp
    const int e = warp - 2;              // 0..15
    const int q = warp & 3;
    const int k = (e >> 2) & 1;
    const int hpar = e >> 3;
    const int tau = k * 128 + q * 32 + lane;
    const int pg = tau >> 4, slot = tau & 15;
    int i = 0;
    // every epilogue warp runs the same loop (named barriers below); after an
    // abort the waits fail fast and the work is skipped
    for (long long u = u0; u < u1; ++u) {
      const int b = (int)(u / a.n_st), st = (int)(u % a.n_st);
      const int t0 = st * kSuper;
      const int len = min(a.seq_lens[b], a.max_pages * kPage);
      if (t0 >= len) continue;
      const int t = t0 + tau;
      const bool valid = t < len;
      for (int it = 0; it < a.n_items; ++it, ++i) {
        const ScoreItem& item = items_s[it];
        const int nh = item.nh;
        const int ks = i % a.KS;
        const bool ok1 = tc::mbar_wait_ab(&k_full[ks], ((uint32_t)(i / a.KS)) & 1u, a.status, &abort_flag);
        const bool ok = ok1 && tc::mbar_wait_ab(&acc_full[i & 1], ((uint32_t)(i >> 1)) & 1u, a.status, &abort_flag);
        tc::tc_fence_after();
        const uint8_t* page = K_s + (size_t)ks * a.k_stage + (size_t)pg * item.key_bytes;
        const uint32_t tcol = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((i & 1) * 256 + k * 128);
        for (int hh = hpar; hh < nh; hh += 2) {
          const HeadPlan& hp = hp_s[item.h0 + hh];
          const uint8_t* blk = page + hp.blk_rel;
          float s = 0.f;
          if (ok) {
            for (int gi = 0; gi < hp.ng; ++gi) {
              const int4 gd = hp.grp[gi];     // start, n, bits, code_off
              const int nf = gd.y >> 3, tail = gd.y & 7;
              float G[32], T[6];
              const uint32_t c0 = tcol + (uint32_t)(hp.hcol + gd.x);
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < nf) tmem_ld8_nw(c0 + 8 * c, G + 8 * c);
              const uint32_t ct = c0 + (uint32_t)(8 * nf);
              if (tail > 0) tmem_ld2_nw(ct, T);
              if (tail > 2) tmem_ld2_nw(ct + 2, T + 2);
              if (tail > 4) tmem_ld2_nw(ct + 4, T + 4);
              tmem_wait(G, T);
              const float scale = __half2float(reinterpret_cast<const __half*>(blk)[gi * kPage + slot]);
              const uint8_t* codes = blk + gd.w;
              const uint32_t bit0 = (uint32_t)(slot * gd.y * gd.z);
              float d;
              if (gd.z == 3)
                d = group_dot<3>(codes, bit0, nf, tail, G, T);
              else if (gd.z == 4)
                d = group_dot<4>(codes, bit0, nf, tail, G, T);
              else
                d = 0.f;     // layers with other code widths do not take this kernel
              s = fmaf(scale, d, s);
            }
          }
          sc_s[hh >> 1][e * 32 + lane] = s;
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&acc_free[i & 1]);
          tc::mbar_arrive(&k_empty[ks]);
        }
        const size_t hb = (size_t)b * a.H + item.h0;
        if (a.S_dbg) {
          for (int hh = hpar; hh < nh; hh += 2)
            if (valid) a.S_dbg[(hb + hh) * a.P_ld + t] = sc_s[hh >> 1][e * 32 + lane];
          continue;
        }
        // softmax statistics per 32-token group (this warp's tokens), per head:
        // m = max s, P = exp2(s - m) rounded to fp16, l = sum of the fp16 P
        const int grp = (t0 >> 5) + k * 4 + q;
        for (int hh = hpar; hh < nh; hh += 2) {
          const float sv = sc_s[hh >> 1][e * 32 + lane];
          float m = valid ? sv : -FLT_MAX;
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          float p = 0.f;
          if (valid) {
            const __half pb = __float2half_rn(exp2f(sv - m));
            a.P[(hb + hh) * a.P_ld + t] = pb;
            p = __half2float(pb);
          }
          for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
          if (lane == 0) {
            a.m_st[(hb + hh) * a.n_g + grp] = m;
            a.l_st[(hb + hh) * a.n_g + grp] = p;
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// W'' item blocks for every sequence: rows of W'' (grouped by item, zero
// padded to the item's N), 128 columns, K-major with 128-byte swizzle, fp16.
// One block per (sequence, item); a thread writes 8 columns of one row.
__global__ void __launch_bounds__(512) k_qprep_tc(LayerView v, const __nv_bfloat16* __restrict__ q,
                                                  const int32_t* __restrict__ seq_lens,
                                                  const int32_t* __restrict__ q_pos, const float* __restrict__ Bk,
                                                  const int* __restrict__ key_off,
                                                  const ScoreItem* __restrict__ items, long long w_stride,
                                                  uint8_t* __restrict__ W) {
  __shared__ float qs[8][128];
  const int b = blockIdx.x, it = blockIdx.y;
  const ScoreItem item = items[it];
  const int pos = q_pos ? q_pos[b] : seq_lens[b] - 1;
  for (int idx = threadIdx.x; idx < item.nh * 64; idx += blockDim.x) {
    const int hh = idx / 64, p = idx % 64;
    const int h = item.h0 + hh;
    const __nv_bfloat16* qh = q + ((size_t)b * v.H + h) * 128;
    const float a0 = __bfloat162float(qh[p]), b0 = __bfloat162float(qh[p + 64]);
    // angle pos * theta_p reduced modulo 2 pi in double, then a float sincos
    const double ang = (double)pos * exp2(-(2.0 * p / 128.0) * (double)v.rope_log2_theta);
    const double two_pi = 6.283185307179586476925286766559;
    const float red = (float)(ang - two_pi * rint(ang / two_pi));
    float sn, cs;
    sincosf(red, &sn, &cs);
    qs[hh][p] = (a0 * cs - b0 * sn) * v.scale_log2;
    qs[hh][p + 64] = (b0 * cs + a0 * sn) * v.scale_log2;
  }
  __syncthreads();
  uint8_t* blk = W + (size_t)b * w_stride + item.w_off;
  const uint32_t atom = (uint32_t)item.npad * 128u;
  for (int idx = threadIdx.x; idx < item.npad * 8; idx += blockDim.x) {
    const int row = idx >> 3, c = idx & 7;       // 8-column chunk c of the 64 (cos | sin) pairs
    int hh = -1;
    for (int x = 0; x < item.nh; ++x)
      if (row >= item.hcol[x] && row < item.hcol[x] + item.hr[x]) hh = x;
    uint32_t re[4] = {0u, 0u, 0u, 0u}, im[4] = {0u, 0u, 0u, 0u};
    if (hh >= 0) {
      const int h = item.h0 + hh, g = h / v.group_q, j = row - item.hcol[hh];
      const float* B = Bk + ((size_t)key_off[g] + j) * 128 + c * 8;
      const float4 x0 = *reinterpret_cast<const float4*>(B), x1 = *reinterpret_cast<const float4*>(B + 4);
      const float4 y0 = *reinterpret_cast<const float4*>(B + 64), y1 = *reinterpret_cast<const float4*>(B + 68);
      const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const float ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int p = c * 8 + i;
        const float r0 = qs[hh][p] * xs[i] + qs[hh][p + 64] * ys[i];
        const float r1 = qs[hh][p + 1] * xs[i + 1] + qs[hh][p + 65] * ys[i + 1];
        const float i0 = qs[hh][p + 64] * xs[i] - qs[hh][p] * ys[i];
        const float i1 = qs[hh][p + 65] * xs[i + 1] - qs[hh][p + 1] * ys[i + 1];
        const __half2 rh = __floats2half2_rn(r0, r1), ih = __floats2half2_rn(i0, i1);
        re[i / 2] = *reinterpret_cast<const uint32_t*>(&rh);
        im[i / 2] = *reinterpret_cast<const uint32_t*>(&ih);
      }
    }
    const uint32_t o = tc::sw128((uint32_t)row, (uint32_t)c);
    *reinterpret_cast<uint4*>(blk + o) = make_uint4(re[0], re[1], re[2], re[3]);
    *reinterpret_cast<uint4*>(blk + atom + o) = make_uint4(im[0], im[1], im[2], im[3]);
  }
}

// RoPE table: for positions t in tile T (128 rows), row t holds
// [cos(t theta_p) for p < 64 | sin(t theta_p) for p < 64] as fp16, K-major swizzled.
__global__ void k_rope_table(float log2_theta, int n_tiles, uint8_t* __restrict__ E) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)n_tiles * 128 * 64) return;
  const int p = (int)(idx % 64);
  const long long t = idx / 64;
  const int tile = (int)(t / 128), row = (int)(t % 128);
  const double freq = exp2(-(2.0 * p / 128.0) * (double)log2_theta);
  double sn, cs;
  sincos((double)t * freq, &sn, &cs);
  uint8_t* base = E + (size_t)tile * kETileBytes;
  const uint32_t o = tc::sw128((uint32_t)row, (uint32_t)(p >> 3)) + (uint32_t)(p & 7) * 2u;
  *reinterpret_cast<__half*>(base + o) = __float2half_rn((float)cs);
  *reinterpret_cast<__half*>(base + 16384 + o) = __float2half_rn((float)sn);
}

}  // namespace

// Plan the MMA items and size the score kernel's buffers.  Returns false if
// the layer's shape does not fit the tensor-core score kernel.
bool plan_scores_tc(starkv_layer* L) {
  const LayerView& v = L->view;
  const starkv_layer_config& c = L->cfg;
  if (c.dtype != STARKV_BF16 || c.plain || !c.rope || c.head_dim != 128 || !v.quantized) return false;
  if (c.n_heads > 64) return false;
  // the epilogue reads TMEM in pairs of columns: every key group must have an even width
  for (int g = 0; g < v.Hkv; ++g)
    for (int k = 0; k < L->lat[g].n_groups; ++k)
      if (L->grp[L->lat[g].group0 + k].n % 2) return false;
  L->items.clear();
  int w_off = 0, max_key = 0, max_w = 0;
  int h = 0;
  while (h < v.H) {
    ScoreItem it{};
    it.h0 = h;
    int cols = 0;
    while (h < v.H && it.nh < 8) {
      const int r = L->lat[h / v.group_q].width;
      if (cols + r > 128) break;
      it.hr[it.nh] = r;
      it.hcol[it.nh++] = cols;
      cols += r;
      ++h;
    }
    if (it.nh == 0) return false;
    it.npad = (cols + 15) / 16 * 16;
    it.w_off = w_off;
    w_off += it.npad * 256;
    const int g0 = it.h0 / v.group_q, g1 = (it.h0 + it.nh - 1) / v.group_q;
    it.key_off = L->lat[g0].block_off;
    it.key_bytes = L->lat[g1 + 1].block_off - it.key_off;
    max_key = std::max(max_key, it.key_bytes);
    max_w = std::max(max_w, it.npad * 256);
    L->items.push_back(it);
  }
  L->w_stride = w_off;
  L->k_stage = (kSuper / kPage) * max_key + 16;
  L->k_stage = (L->k_stage + 1023) / 1024 * 1024;
  L->w_stage = (max_w + 1023) / 1024 * 1024;
  // dynamic shared memory next to ~21 KB of static tables and barriers
  const size_t budget = 204 * 1024 - 2 * kETileBytes;
  L->WS = 3;
  L->KS = 2;
  while (L->WS > 2 && (size_t)L->WS * L->w_stage + (size_t)L->KS * L->k_stage > budget) --L->WS;
  if ((size_t)L->WS * L->w_stage + (size_t)L->KS * L->k_stage > budget) return false;
  const int mp = c.max_positions > 0 ? c.max_positions : 32768;
  L->rope_tiles = (mp + kSuper - 1) / kSuper * (kSuper / 128);
  return true;
}

cudaError_t build_rope_table(starkv_layer* L, cudaStream_t s) {
  const long long n = (long long)L->rope_tiles * 128 * 64;
  k_rope_table<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L->view.rope_log2_theta, L->rope_tiles,
                                                           (uint8_t*)L->rope_E);
  return cudaGetLastError();
}

size_t scores_tc_ws_bytes(const starkv_layer* L, int batch, int max_len) {
  const int n_st = (max_len + kSuper - 1) / kSuper;
  const size_t P_ld = (size_t)n_st * kSuper;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  return r((size_t)batch * L->w_stride) + r(2 * (size_t)batch * L->view.H * P_ld) +
         2 * r(sizeof(float) * (size_t)batch * L->view.H * (P_ld / 32));
}

cudaError_t launch_scores_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                             void* ws, ScoreOut* out, float* S_dbg, long long S_ld, cudaStream_t s) {
  const LayerView& v = L->view;
  const int max_len = max_pages * kPage;
  const int n_st = (max_len + kSuper - 1) / kSuper;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = (uint8_t*)ws;
  uint8_t* W = w;
  w += r((size_t)batch * L->w_stride);
  out->P_ld = S_dbg ? S_ld : (long long)n_st * kSuper;
  out->n_st = n_st;
  out->P = (__half*)w;
  w += r(2 * (size_t)batch * v.H * n_st * kSuper);
  out->n_g = n_st * (kSuper / 32);
  out->m_st = (float*)w;
  w += r(sizeof(float) * (size_t)batch * v.H * out->n_g);
  out->l_st = (float*)w;
  k_qprep_tc<<<dim3(batch, (unsigned)L->items.size()), 512, 0, s>>>(
      v, (const __nv_bfloat16*)q, seq_lens, q_pos, L->Bk, L->d_key_off, L->d_items, L->w_stride, W);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ScoreArgs a;
  a.pool = pool;
  a.n_pages = n_pages;
  a.page_bytes = (long long)L->page_bytes;
  a.pt = pt;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.E = (const uint8_t*)L->rope_E;
  a.W = W;
  a.w_stride = L->w_stride;
  a.items = L->d_items;
  a.n_items = (int)L->items.size();
  a.lat = L->d_lat;
  a.grp = L->d_grp;
  a.gq = v.group_q;
  a.n_st = n_st;
  a.U = (long long)batch * n_st;
  a.P = out->P;
  a.P_ld = out->P_ld;
  a.m_st = out->m_st;
  a.l_st = out->l_st;
  a.n_g = out->n_g;
  a.S_dbg = S_dbg;
  a.H = v.H;
  a.w_stage = L->w_stage;
  a.k_stage = L->k_stage;
  a.WS = L->WS;
  a.KS = L->KS;
  a.status = L->status;
  const size_t smem = 2 * kETileBytes + (size_t)a.WS * a.w_stage + (size_t)a.KS * a.k_stage + 1024;
  static size_t attr = 0;
  if (smem > attr) {
    e = cudaFuncSetAttribute(k_scores_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  const int G = (int)std::min<long long>(num_sms(), a.U);
  k_scores_tc<<<G, kScoreThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace starkv
