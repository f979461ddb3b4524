// Joint-value contraction on tcgen05 tensor cores ("STAR-KV 阅读笔记"
// section 5.3 and Algorithm 2 step 6: stack the heads' probabilities and
// multiply them by the shared low-rank value latent in one matrix product).
//
//     Y_h = sum_t p_h(t) zhat_v(t)       for all query heads h at once
//
// computed transposed, Y^T = Zv^T P^T: the dequantized value latent of one
// 16-token page is the A operand (M = 128 value channels per block, K = the
// page's 16 tokens), the stacked probabilities are B (N = heads, K-major in
// shared memory), and Y^T for every 128-channel block stays in TMEM for a
// whole run of pages.  The A tiles never touch shared memory: the value
// latent's codes are stored channel-major, so a thread that owns one channel
// (one TMEM lane) finds that channel's 16 codes in one field, turns them into
// fp16 token pairs in registers and stores them straight into TMEM, where the
// MMA reads A.
//
// An M = 128, N = 32 MMA does little work per instruction, and one thread
// cannot issue tcgen05.mma much faster than one every ~50 cycles, so the MMAs
// are issued by four threads on the four schedulers: the 16 dequantizing
// warps form four teams (one warp per TMEM lane quarter each), team j owns
// the channel blocks j, j + 4, ... with their own ring of A slots in TMEM, and
// the team's own MMA warp issues its MMAs once the four have stored a page,
// while they go on to the next page.  Teams meet only at the shared page
// copies and P tiles.
//
// P comes from the score kernel as exp2(s - m_g) per 32-token group; it is
// rescaled by exp2(m_g - M) with M the maximum over the CTA's run of the
// sequence, so no accumulator ever needs rescaling.  The CTA writes one
// partial (M, l, Y) per run of one sequence; a combine kernel merges the runs.
//   warp 0      bulk copies of the pages' value blocks, TMEM allocation
//   warps 1-4   P staging: rescaled fp16 P tiles (the B operand), M and l;
//               warp s takes the 32-token group s of every 128-token tile
//   warps 5-8   MMA issue, one warp (lane 0) per team, on four schedulers
//   warps 9-24  four teams of four workers: dequantize the team's channel
//               groups of each page into its A slot, read its blocks of Y^T
//               at the end of a run
#include <float.h>

#include "tc_common.cuh"

namespace starkv {

namespace {

constexpr int kTeams = 4;                                // MMA-issuing teams, four warps each
constexpr int kValWorkers = 4 * kTeams;                  // dequantizing warps
constexpr int kStagers = 4;                              // P staging warps, one per 32-token group of a tile
constexpr int kIssuer0 = 1 + kStagers;                   // first MMA warp (one per team)
constexpr int kWorker0 = kIssuer0 + kTeams;              // first worker warp
constexpr int kValThreads = 32 * (kWorker0 + kValWorkers);   // page copies, P staging, MMA, workers
constexpr int kMaxRawStages = 32;
constexpr int kMaxASlots = 8;    // A slots (two pages each) a team keeps in TMEM at once
constexpr int kVSuper = 256;     // tokens per super-tile (matches the score kernel)
constexpr int kMaxRuns = 64;     // runs (sequences) per CTA
constexpr int kRunMaxCache = 16; // runs whose per-head maxima are computed up front
constexpr int kMaxTiles = 256;   // 128-token tiles per CTA

// Atomic maximum of floats (no NaN) through their integer orderings.
__device__ __forceinline__ void atomic_max_float(float* addr, float v) {
  if (v >= 0.f)
    atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
  else
    atomicMin(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

struct ValArgs {
  const uint8_t* pool;
  long long n_pages, page_bytes;
  const int32_t* pt;
  int max_pages;
  const int32_t* seq_lens;
  int vblk_off, vblk_bytes;     // value latent block inside a page
  int raw_stage;                // bytes of one raw stage (a page's value block, 128-byte aligned)
  int n_raw;                    // raw stages
  int na;                       // A slots of each team in TMEM
  const GroupDesc* vgrp;        // value latent groups (all of 32 channels)
  int rv, H;
  int lg_nblk;                  // log2 of the 128-channel blocks of the value latent
  const __half* P;              // [B][H][P_ld]
  long long P_ld;
  const float* m_st;            // [B][H][n_g]: maximum of each 32-token group
  int n_st;
  int n_g;
  long long U;                  // batch * n_st; unit u = (sequence u / n_st, super-tile u % n_st)
  int slots;                    // partial slots per CTA
  float* Y;                     // [G][slots][H][rv]
  float* mseg;                  // [G][slots][H]
  float* lseg;
  uint32_t* status;
};

__device__ __forceinline__ long long vunit_lo(int c, int G, long long U) { return (long long)c * U / G; }

// Two fp16 lanes holding 1024 + u (an exact fp16 integer: the code in the
// low mantissa bits of 0x6400) -> (u - 2^(B-1)) * scale: one exact
// subtraction of 1024 + 2^(B-1), one correctly rounded multiply by the
// token's fp16 scale.
__device__ __forceinline__ uint32_t deq_pair(uint32_t x, __half2 sub, uint32_t scales) {
  __half2 h = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&x), sub),
                      *reinterpret_cast<const __half2*>(&scales));
  return *reinterpret_cast<uint32_t*>(&h);
}

// One channel's 16 codes (its field of a channel-major code block) -> eight
// fp16 pairs, pair c = tokens (2c, 2c + 1) of the page, the layout of one
// 128 x 16 A tile row in TMEM.  The field holds the even slots first, then
// the odd slots, so each pair comes out of one shift and mask.
//   4-bit: word 0 = slots 0 2 4 .. 14, word 1 = slots 1 3 .. 15 (a nibble each);
//          byte j of both words, side by side, gives pairs 2j and 2j + 1.
//   3-bit: 48 bits, slots 0 2 .. 14 at bits 0-23, slots 1 3 .. 15 at 24-47;
//          pair c sits at bits 3c and 24 + 3c.
__device__ __forceinline__ void deq_channel4(uint32_t w0, uint32_t w1, __half2 sub, const uint32_t* sc,
                                             uint32_t* out) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t r = __byte_perm(w0, w1, (uint32_t)j | ((uint32_t)(4 + j) << 8));
    out[2 * j] = deq_pair((r & 0x000F000Fu) | 0x64006400u, sub, sc[2 * j]);
    out[2 * j + 1] = deq_pair(((r >> 4) & 0x000F000Fu) | 0x64006400u, sub, sc[2 * j + 1]);
  }
}
__device__ __forceinline__ void deq_channel3(uint64_t x, __half2 sub, const uint32_t* sc, uint32_t* out) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    // codes at bits 0-2 and 24-26 -> bytes 0 and 2, 0x64 into bytes 1 and 3
    const uint32_t t = (uint32_t)(x >> (3 * c)) & 0x07000007u;
    out[c] = deq_pair(__byte_perm(t, 0x64646464u, 0x4340u), sub, sc[c]);
  }
}

// An unquantized bf16 value latent is stored channel-major too: channel j's
// 16 tokens are 32 contiguous bytes.  Word c holds slots 2c and 2c + 1, which
// become one fp16 pair of the A tile row (bf16 -> fp32 is exact, fp32 -> fp16
// rounds to nearest; the latents are far inside the fp16 range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// NBT: 128-channel blocks per team (the value latent has 128 * nblk channels,
// team j owns blocks j + 4 i, i < NBT).  BF16: the value latent is unquantized
// bf16 instead of 4/3-bit codes.
template <int NBT, bool BF16>
__global__ void __launch_bounds__(kValThreads, 1) k_values_tc(ValArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t t_full[kTeams][kMaxASlots], t_free[kTeams][kMaxASlots], t_seg[kTeams],
      t_acc[kTeams], r_full[kMaxRawStages], r_empty[kMaxRawStages];
  __shared__ __align__(8) uint64_t p_full[2], p_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ int4 vg_s[128];              // per value group: code width, code block offset, fp16x2 of 1024 + 2^(bits-1)
  __shared__ int4 tile_s[kMaxTiles];      // per tile: sequence, first token, length, run
  __shared__ int pid_s[kMaxTiles][8];     // per tile: page of each 16-token slot block
  __shared__ uint8_t rsp_s[kMaxTiles * 8];   // per page of the CTA: raw stage | phase parity << 7
  __shared__ int run_b[kMaxRuns];
  __shared__ int n_tiles_s, n_runs_s;
  __shared__ float l_part[kStagers][64];  // per stager warp and head: its part of the run sum of the staged P
  __shared__ float runM_s[kRunMaxCache][64];   // per run and head: the maximum of the 32-token group maxima
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* P_s = smem;                                   // 2 x (H x 128 fp16, K-major swizzled)
  uint8_t* R_s = P_s + 2 * a.H * 256;                    // n_raw raw stages
  const int p_stage = a.H * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const long long u0 = vunit_lo(cta, G, a.U), u1 = vunit_lo(cta + 1, G, a.U);
  const int nblk = 1 << a.lg_nblk;                       // 128-channel blocks
  const int n_teams = min(kTeams, nblk);                 // teams with blocks
  const uint32_t ycols = (uint32_t)(nblk * a.H);         // TMEM columns of Y^T; the teams' A rings follow
  const int b_first = (int)(u0 / a.n_st);

  if (threadIdx.x == 0) {
    for (int t = 0; t < kTeams; ++t) {
      for (int s = 0; s < a.na; ++s) {
        tc::mbar_init(&t_full[t][s], 4);
        tc::mbar_init(&t_free[t][s], 1);
      }
      tc::mbar_init(&t_seg[t], 1);
      tc::mbar_init(&t_acc[t], 4);
    }
    for (int s = 0; s < a.n_raw; ++s) {
      tc::mbar_init(&r_full[s], 1);
      tc::mbar_init(&r_empty[s], 4 * n_teams);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&p_full[s], kStagers);
      tc::mbar_init(&p_empty[s], n_teams);
    }
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  for (int g = threadIdx.x; g < (BF16 ? 0 : a.rv / 32); g += blockDim.x) {
    const int bits = a.vgrp[g].bits;
    const float offm = 1024.f + (float)(1 << (bits - 1));
    const __half2 sub = __floats2half2_rn(offm, offm);
    vg_s[g] = make_int4(bits, a.vgrp[g].code_off, *reinterpret_cast<const int*>(&sub), 0);
  }
  if (warp == 0) {
    // tile table: 32 units at a time, tiles placed by a warp prefix count
    int nt = 0, nr = 0, last_b = -1;
    for (long long ub = u0; ub < u1; ub += 32) {
      const long long u = ub + lane;
      int b = 0, st = 0, len = 0, ntl = 0;
      if (u < u1) {
        b = (int)(u / a.n_st);
        st = (int)(u - (long long)b * a.n_st);
        len = min(a.seq_lens[b], a.max_pages * kPage);
        ntl = (st * kVSuper < len) + (st * kVSuper + 128 < len);
      }
      int pre = ntl;   // inclusive prefix sum of tile counts
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += y;
      }
      // run index: a new run starts at each unit with tiles whose sequence differs from the previous such unit's
      const unsigned has = __ballot_sync(0xffffffffu, ntl > 0);
      const int prev_lane = 31 - __clz(has & ((1u << lane) - 1u));   // -1 when none
      const int prev_b = __shfl_sync(0xffffffffu, b, prev_lane < 0 ? 0 : prev_lane);
      const bool starts = ntl > 0 && (prev_lane < 0 ? b != last_b : b != prev_b);
      const unsigned st_mask = __ballot_sync(0xffffffffu, starts);
      const int run = nr + __popc(st_mask & ((2u << lane) - 1u)) - 1;
      if (starts && run < kMaxRuns) run_b[run] = b;
      for (int k = 0; k < ntl; ++k) {
        const int T = nt + pre - ntl + k;
        if (T < kMaxTiles) tile_s[T] = make_int4(b, st * kVSuper + k * 128, len, run);
      }
      nt += __shfl_sync(0xffffffffu, pre, 31);
      nr += __popc(st_mask);
      if (has) last_b = __shfl_sync(0xffffffffu, b, 31 - __clz(has));
    }
    if (lane == 0) {
      n_tiles_s = min(nt, kMaxTiles);
      n_runs_s = min(nr, kMaxRuns);
    }
    tc::tmem_alloc(&tmem_base, 512);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int n_tiles = n_tiles_s;
  // page ids of every tile (out-of-range entries set the status bit and read page 0)
  for (int e = threadIdx.x; e < n_tiles * 8; e += blockDim.x) {
    const int4 tl = tile_s[e >> 3];
    const int t = tl.y + (e & 7) * kPage;
    int page = -1;
    if (t < tl.z) {
      page = a.pt[(size_t)tl.x * a.max_pages + t / kPage];
      if (page < 0 || page >= a.n_pages) {
        atomicOr(a.status, kBadPage);
        page = 0;
      }
    }
    pid_s[e >> 3][e & 7] = page;
    rsp_s[e] = (uint8_t)((e % a.n_raw) | (((e / a.n_raw) & 1) << 7));
  }
  for (int x = threadIdx.x; x < kRunMaxCache * 64; x += blockDim.x) (&runM_s[0][0])[x] = -FLT_MAX;
  __syncthreads();
  // run maxima, all threads at once (a tile contributes its four groups)
  for (int e = threadIdx.x; e < n_tiles * a.H; e += blockDim.x) {
    const int T = e / a.H, h = e - T * a.H;
    const int4 tl = tile_s[T];
    if (tl.w < kRunMaxCache) {
      const float4 g4 = *reinterpret_cast<const float4*>(a.m_st + ((size_t)tl.x * a.H + h) * a.n_g + (tl.y >> 5));
      atomic_max_float(&runM_s[tl.w][h], fmaxf(fmaxf(g4.x, g4.y), fmaxf(g4.z, g4.w)));
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------ page copies
    // Page p = 8 T + k (tokens 16 k .. 16 k + 15 of tile T): its value block
    // into raw stage p % n_raw.
    if (lane == 0) {
      const int n_pg = n_tiles * 8;
      int issued = 0;
      for (int pg = 0; pg < n_pg; ++pg) {
        const uint32_t rsp = rsp_s[pg];
        const int rs = (int)(rsp & 127u);
        if (!tc::mbar_wait_ab_lazy(&r_empty[rs], (rsp >> 7) ^ 1u, a.status, &abort_flag)) break;
        const int page = pid_s[pg >> 3][pg & 7];
        tc::mbar_expect_tx(&r_full[rs], page >= 0 ? (uint32_t)a.vblk_bytes : 0u);
        if (page >= 0)
          tc::bulk_g2s(R_s + (size_t)rs * a.raw_stage, a.pool + (size_t)page * a.page_bytes + a.vblk_off,
                       (uint32_t)a.vblk_bytes, &r_full[rs]);
        issued = pg + 1;
      }
      // let copies in flight land before the CTA can exit
      for (int pg = max(0, issued - a.n_raw); pg < issued; ++pg)
        tc::mbar_wait(&r_full[pg % a.n_raw], ((uint32_t)(pg / a.n_raw)) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp <= kStagers) {
    // ------------------------------------------------ P staging
    // Stager warp s stages the 32-token group s of every tile, lane h for
    // head h (and h + 32): P * exp2(m_g - M) rounded to fp16, with M the
    // maximum over the run; l = sum of the staged values, added in a fixed
    // order over the four stagers.
    const int sw = warp - 1;
    if (sw == 0)
      for (int sl = 0; sl < a.slots; ++sl)
        for (int h = lane; h < a.H; h += 32) {
          a.mseg[((size_t)cta * a.slots + sl) * a.H + h] = -FLT_MAX;
          a.lseg[((size_t)cta * a.slots + sl) * a.H + h] = 0.f;
        }
    float Mh[2] = {-FLT_MAX, -FLT_MAX}, lh[2] = {0.f, 0.f};
    int cur_run = -1, cur_b = -1;
    auto flush = [&]() {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        if (lane + 32 * hh < a.H) l_part[sw][lane + 32 * hh] = lh[hh];
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kStagers) : "memory");
      if (sw == 0) {
        const size_t base = ((size_t)cta * a.slots + (cur_b - b_first)) * a.H;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = lane + 32 * hh;
          if (h < a.H) {
            a.mseg[base + h] = Mh[hh];
            a.lseg[base + h] = ((l_part[0][h] + l_part[1][h]) + l_part[2][h]) + l_part[3][h];
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kStagers) : "memory");
    };
    for (int T = 0; T < n_tiles; ++T) {
      const int4 tl = tile_s[T];   // sequence, first token, length, run
      if (tl.w != cur_run) {
        if (cur_run >= 0) flush();
        cur_run = tl.w;
        cur_b = tl.x;
        // the run maximum over its tiles' 32-token groups
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = lane + 32 * hh;
          float m = -FLT_MAX;
          if (h < a.H && tl.w < kRunMaxCache) {
            m = runM_s[tl.w][h];
          } else if (h < a.H) {
            const float* mr = a.m_st + ((size_t)tl.x * a.H + h) * a.n_g;
            for (int T2 = T; T2 < n_tiles && tile_s[T2].w == tl.w; ++T2) {
              const float4 g4 = *reinterpret_cast<const float4*>(mr + (tile_s[T2].y >> 5));
              m = fmaxf(m, fmaxf(fmaxf(g4.x, g4.y), fmaxf(g4.z, g4.w)));
            }
          }
          Mh[hh] = m;
          lh[hh] = 0.f;
        }
      }
      const int t0 = tl.y + 32 * sw;   // this warp's 32 tokens
      // loads first, then the wait for the stage
      uint4 raw[2][4];
      float mg[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = lane + 32 * hh;
        mg[hh] = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) raw[hh][c8] = make_uint4(0, 0, 0, 0);
        if (h < a.H && t0 < tl.z) {
          const size_t row = (size_t)tl.x * a.H + h;
          mg[hh] = a.m_st[row * a.n_g + (t0 >> 5)];
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8)
            if (t0 + c8 * 8 < tl.z) raw[hh][c8] = *reinterpret_cast<const uint4*>(a.P + row * a.P_ld + t0 + c8 * 8);
        }
      }
      const int ps = T & 1;
      if (!tc::mbar_wait_ab(&p_empty[ps], (((uint32_t)(T >> 1)) & 1u) ^ 1u, a.status, &abort_flag)) break;
      uint8_t* pt_s = P_s + (size_t)ps * p_stage;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = lane + 32 * hh;
        if (h >= a.H) continue;
        const float f = t0 < tl.z ? exp2f(mg[hh] - Mh[hh]) : 0.f;
        float lsum = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {   // 8-token chunks
          const int ch = sw * 4 + c8;
          const int tp = t0 + c8 * 8;
          __half* hv = reinterpret_cast<__half*>(&raw[hh][c8]);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float p = (tp + i < tl.z) ? __half2float(hv[i]) * f : 0.f;
            hv[i] = __float2half_rn(p);
            lsum += __half2float(hv[i]);
          }
          *reinterpret_cast<uint4*>(pt_s + (ch >> 3) * (a.H * 128) + tc::sw128((uint32_t)h, (uint32_t)(ch & 7))) =
              raw[hh][c8];
        }
        lh[hh] += lsum;
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[ps]);
    }
    if (cur_run >= 0) flush();
  } else if (warp < kWorker0) {
    // ------------------------------------------------ MMA issue, one warp per team
    // Team j's pages 2 m and 2 m + 1 sit in its A slot m % na: block j + 4 i's
    // 128 x 16 A tile of page e at TMEM column abase + (slot NBT + i) 16 + 8 e;
    // its K = 16 MMA adds that block's Y^T (columns (j + 4 i) H ..).  At the
    // end of a run the warp commits t_seg and waits for the team to have read
    // Y^T (t_acc) before the next run's first MMA overwrites it.
    const int j = warp - kIssuer0;
    if (j < n_teams && lane == 0) {
      const int nbt = min(NBT, (nblk - j + 3) / 4);
      const uint32_t abase = ycols + (uint32_t)(j * a.na * NBT * 16);
      const uint32_t idesc = tc::idesc_f16(128, a.H, false, false, false);
      const uint64_t b0 = tc::sdesc_sw128(tc::smem_u32(P_s), 0, 1024);   // B: K-major, 64-token atoms of H rows
      const uint32_t b_lo0 = tc::desc_lo(b0), b_hi = tc::desc_hi(b0);
      const uint32_t b_atom = (uint32_t)(a.H * 128) >> 4, p_step = (uint32_t)p_stage >> 4;
      int cur_run = -1, n_runs_done = 0, as = 0;
      uint32_t aph = 0;
      bool first = false;
      for (int T = 0; T < n_tiles && !abort_flag; ++T) {
        const int run = tile_s[T].w;
        if (run != cur_run) {
          if (cur_run >= 0) {
            tc::mma_commit(&t_seg[j]);
            if (!tc::mbar_wait_ab(&t_acc[j], (uint32_t)n_runs_done & 1u, a.status, &abort_flag)) break;
            ++n_runs_done;
            tc::tc_fence_after();
          }
          cur_run = run;
          first = true;
        }
        const int ps = T & 1;
        if (!tc::mbar_wait_ab(&p_full[ps], ((uint32_t)(T >> 1)) & 1u, a.status, &abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t b_lo = b_lo0 + (uint32_t)ps * p_step;
        bool ok = true;
        for (int k = 0; k < 8; k += 2) {
          if (!tc::mbar_wait_ab(&t_full[j][as], aph, a.status, &abort_flag)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t acol = tmem + abase + (uint32_t)(as * NBT * 16);
          const uint32_t bk = b_lo + (uint32_t)(k >> 2) * b_atom + (uint32_t)(k & 3) * 2u;   // pages k, k + 1: K steps
          const uint32_t acc = (first && k == 0) ? 0u : 1u;
#pragma unroll
          for (int i = 0; i < NBT; ++i) {
            if (i >= nbt) break;
            const uint32_t dcol = tmem + (uint32_t)((j + 4 * i) * a.H);
            tc::mma_f16_ts(dcol, acol + (uint32_t)i * 16u, bk, b_hi, idesc, acc);
            tc::mma_f16_ts(dcol, acol + (uint32_t)i * 16u + 8u, bk + 2u, b_hi, idesc, 1u);
          }
          tc::mma_commit(&t_free[j][as]);
          if (++as == a.na) {
            as = 0;
            aph ^= 1u;
          }
        }
        if (!ok) break;
        tc::mma_commit(&p_empty[ps]);
        first = false;
      }
      if (cur_run >= 0) tc::mma_commit(&t_seg[j]);
      // every MMA of this thread has completed before the CTA may exit
      tc::mma_commit(&t_free[j][as]);
      tc::mbar_wait(&t_free[j][as], aph, a.status);
    }
  } else {
    // ------------------------------------------------ worker teams
    // A warp may address only its TMEM lane quarter q = warp % 4, i.e. the
    // channels 32 q .. 32 q + 31 of every 128-channel block: channel group
    // 4 cb + q of block cb, lane = channel inside the group.  Team j = the
    // four consecutive workers (one per quarter) owning blocks j + 4 i.
    const int wid = warp - kWorker0;
    const int q = warp & 3, j = wid >> 2;
    if (j < n_teams) {
      const uint32_t lane_base = (uint32_t)(q * 32) << 16;
      const uint32_t abase = ycols + (uint32_t)(j * a.na * NBT * 16);   // this team's A ring (slots of two pages)
      const int nbt = min(NBT, (nblk - j + 3) / 4);                    // blocks of this team
      const int n_pg = n_tiles * 8;
      int cur_run = -1, n_epi = 0, as = 0;
      uint32_t aph = 0;
      auto epilogue = [&](int r) {
        // Y^T of this team's blocks for run r (lanes = value channels), 16 columns at a time
        const bool ok = tc::mbar_wait_ab(&t_seg[j], (uint32_t)n_epi & 1u, a.status, &abort_flag);
        ++n_epi;
        tc::tc_fence_after();
        const size_t base = ((size_t)cta * a.slots + (run_b[r] - b_first)) * a.H;
#pragma unroll
        for (int i = 0; i < NBT; ++i) {
          if (i >= nbt) break;
          const int cb = j + 4 * i;
          const int ch = cb * 128 + q * 32 + lane;
          for (int h0 = 0; h0 < a.H; h0 += 16) {
            float v[16];
            if (ok) {
              tc::tmem_ld16_sync(tmem + lane_base + (uint32_t)(cb * a.H + h0), v);
            } else {
#pragma unroll
              for (int x = 0; x < 16; ++x) v[x] = 0.f;
            }
#pragma unroll
            for (int x = 0; x < 16; ++x) a.Y[(base + h0 + x) * a.rv + ch] = v[x];
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&t_acc[j]);   // the MMA warp may overwrite Y^T
      };
      for (int p = 0; p < n_pg; p += 2) {
        // pages p and p + 1 (same tile, same run) go into one A slot
        const int T = p >> 3, k = p & 7;
        const int run = tile_s[T].w;
        if (run != cur_run) {
          if (cur_run >= 0) epilogue(cur_run);
          cur_run = run;
        }
        const int cur_as = as;
        const uint32_t cur_aph = aph;
        if (++as == a.na) {
          as = 0;
          aph ^= 1u;
        }
        const uint32_t rsp0 = rsp_s[p], rsp1 = rsp_s[p + 1];
        const int rs0 = (int)(rsp0 & 127u), rs1 = (int)(rsp1 & 127u);
        const bool valid0 = pid_s[T][k] >= 0, valid1 = pid_s[T][k + 1] >= 0;
        const uint32_t slot_col = abase + (uint32_t)(cur_as * NBT * 16);
        const bool ok = tc::mbar_wait_ab(&t_free[j][cur_as], cur_aph ^ 1u, a.status, &abort_flag) &&
                        tc::mbar_wait_ab(&r_full[rs0], rsp0 >> 7, a.status, &abort_flag) &&
                        tc::mbar_wait_ab(&r_full[rs1], rsp1 >> 7, a.status, &abort_flag);
        if (ok) {
#pragma unroll
          for (int i = 0; i < NBT; ++i) {
            if (i >= nbt) break;
            const int g = (j + 4 * i) * 4 + q;
            if constexpr (BF16) {
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const uint8_t* row = R_s + (size_t)(e ? rs1 : rs0) * a.raw_stage + (size_t)(g * 32 + lane) * 32;
                uint32_t out[8];
                if (e ? valid1 : valid0) {
                  const uint4 w0 = *reinterpret_cast<const uint4*>(row);
                  const uint4 w1 = *reinterpret_cast<const uint4*>(row + 16);
                  out[0] = bf16x2_to_f16x2(w0.x); out[1] = bf16x2_to_f16x2(w0.y);
                  out[2] = bf16x2_to_f16x2(w0.z); out[3] = bf16x2_to_f16x2(w0.w);
                  out[4] = bf16x2_to_f16x2(w1.x); out[5] = bf16x2_to_f16x2(w1.y);
                  out[6] = bf16x2_to_f16x2(w1.z); out[7] = bf16x2_to_f16x2(w1.w);
                } else {
#pragma unroll
                  for (int x = 0; x < 8; ++x) out[x] = 0u;
                }
                tc::tmem_st8(tmem + lane_base + slot_col + (uint32_t)(i * 16 + e * 8), out);
              }
              continue;
            }
            const int4 vg = vg_s[g];
            const __half2 sub = *reinterpret_cast<const __half2*>(&vg.z);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint8_t* blk = R_s + (size_t)(e ? rs1 : rs0) * a.raw_stage;
              const bool valid = e ? valid1 : valid0;
              uint32_t sc[8], out[8];
              if (valid) {
                const uint4 s0 = *reinterpret_cast<const uint4*>(blk + g * 32);
                const uint4 s1 = *reinterpret_cast<const uint4*>(blk + g * 32 + 16);
                sc[0] = s0.x; sc[1] = s0.y; sc[2] = s0.z; sc[3] = s0.w;
                sc[4] = s1.x; sc[5] = s1.y; sc[6] = s1.z; sc[7] = s1.w;
              } else {
#pragma unroll
                for (int x = 0; x < 8; ++x) sc[x] = 0u;
              }
              if (vg.x == 4) {
                const uint2 cw = *reinterpret_cast<const uint2*>(blk + vg.y + lane * 8);
                deq_channel4(cw.x, cw.y, sub, sc, out);
              } else {
                const int bit = 48 * lane;
                const uint32_t* cw = reinterpret_cast<const uint32_t*>(blk + vg.y) + (bit >> 5);
                const uint64_t x = ((uint64_t)cw[1] << 32 | cw[0]) >> (bit & 31);
                deq_channel3(x, sub, sc, out);
              }
              tc::tmem_st8(tmem + lane_base + slot_col + (uint32_t)(i * 16 + e * 8), out);
            }
          }
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&t_full[j][cur_as]);
          tc::mbar_arrive(&r_empty[rs0]);
          tc::mbar_arrive(&r_empty[rs1]);
        }
      }
      if (cur_run >= 0) epilogue(cur_run);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// Merge the runs of each sequence: y = sum exp2(M_r - M) Y_r / sum exp2(M_r - M) l_r,
// written as fp16 B-operand tiles of the output kernel.
__global__ void k_values_combine(const float* __restrict__ Y, const float* __restrict__ mseg,
                                 const float* __restrict__ lseg, int G, long long U, int n_st, int slots, int H,
                                 int rv, int NB, int KT, uint8_t* __restrict__ ytiles) {
  // The runs of sequence b are the partial slots of the CTAs whose unit
  // ranges meet [b n_st, (b + 1) n_st).  Candidates c_lo, c_lo + 1, ... are
  // tested one per thread, with their (M, l) read in parallel; a candidate
  // that holds none of the sequence, or whose run saw no valid token, gets
  // weight 0 and its Y is never read.
  constexpr int kCand = 512;
  __shared__ int seg_i[kCand];
  __shared__ float seg_m[kCand], seg_w[kCand];
  __shared__ float red_s[32];
  __shared__ float bmax, inv_den;
  const int b = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  const long long lo = (long long)b * n_st, hi = lo + n_st;
  const int c_lo = max(0, (int)((lo * G) / U) - 1);
  const int c_hi = min(G, (int)((hi * G + U - 1) / U) + 1);
  const int nc = min(c_hi - c_lo, kCand);
  float m = -FLT_MAX;
  for (int t = threadIdx.x; t < nc; t += blockDim.x) {
    const int c = c_lo + t;
    const long long b0 = vunit_lo(c, G, U), b1 = vunit_lo(c + 1, G, U);
    int ik = 0;
    float mk = -FLT_MAX, lk = 0.f;
    if (b1 > b0 && b1 > lo && b0 < hi) {
      ik = (c * slots + (b - (int)(b0 / n_st))) * H + h;
      lk = lseg[ik];
      mk = lk > 0.f ? mseg[ik] : -FLT_MAX;
    }
    seg_i[t] = ik;
    seg_m[t] = mk;
    seg_w[t] = lk;
    m = fmaxf(m, mk);
  }
  // block maximum of M over the runs with l > 0
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red_s[wid] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float x = -FLT_MAX;
    for (int w = 0; w < nw; ++w) x = fmaxf(x, red_s[w]);
    bmax = x;
  }
  __syncthreads();
  const float M = bmax;
  // weights exp2(M_r - M) and the denominator sum w_r l_r
  float dn = 0.f;
  for (int t = threadIdx.x; t < nc; t += blockDim.x) {
    const float l = seg_w[t];
    const float w = l > 0.f ? exp2f(seg_m[t] - M) : 0.f;
    seg_w[t] = w;
    dn += w * l;
  }
  for (int o = 16; o > 0; o >>= 1) dn += __shfl_xor_sync(0xffffffffu, dn, o);
  if (lane == 0) red_s[wid] = dn;
  __syncthreads();
  if (threadIdx.x == 0) {
    float den = 0.f;
    for (int w = 0; w < nw; ++w) den += red_s[w];
    inv_den = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  const float idn = inv_den;
  const int nt = b / NB, r = b % NB;
  // four channels per thread, one 16-byte load per run
  for (int j = 4 * (int)threadIdx.x; j < rv; j += 4 * (int)blockDim.x) {
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    int k = 0;
    for (; k + 2 <= nc; k += 2) {
      const float w0 = seg_w[k], w1 = seg_w[k + 1];
      const float4 y0 = w0 != 0.f ? *reinterpret_cast<const float4*>(Y + (size_t)seg_i[k] * rv + j) : a1;
      const float4 y1 = w1 != 0.f ? *reinterpret_cast<const float4*>(Y + (size_t)seg_i[k + 1] * rv + j) : a1;
      a0.x += w0 * y0.x;
      a0.y += w0 * y0.y;
      a0.z += w0 * y0.z;
      a0.w += w0 * y0.w;
      a1.x += w1 * y1.x;
      a1.y += w1 * y1.y;
      a1.z += w1 * y1.z;
      a1.w += w1 * y1.w;
    }
    if (k < nc && seg_w[k] != 0.f) {
      const float w0 = seg_w[k];
      const float4 y0 = *reinterpret_cast<const float4*>(Y + (size_t)seg_i[k] * rv + j);
      a0.x += w0 * y0.x;
      a0.y += w0 * y0.y;
      a0.z += w0 * y0.z;
      a0.w += w0 * y0.w;
    }
    const __half2 lo2 = __floats2half2_rn((a0.x + a1.x) * idn, (a0.y + a1.y) * idn);   // channels j, j + 1
    const __half2 hi2 = __floats2half2_rn((a0.z + a1.z) * idn, (a0.w + a1.w) * idn);   // channels j + 2, j + 3
    const uint32_t kk = (uint32_t)(h * rv + j), cidx = kk & 63u;
    uint8_t* tile = ytiles + ((size_t)nt * KT + (kk >> 6)) * (size_t)NB * 128;
    const uint32_t off = tc::sw128((uint32_t)r, cidx >> 3) + (cidx & 7u) * 2u;
    *reinterpret_cast<uint2*>(tile + off) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo2), *reinterpret_cast<const uint32_t*>(&hi2));
  }
}

}  // namespace

// Dynamic shared memory of the value kernel: two P stages and the raw page stages.
static size_t values_raw_stage(int vblk_bytes) { return (size_t)(vblk_bytes + 127) / 128 * 128; }
static size_t values_smem(int H, int vblk_bytes, int n_raw) {
  return 2 * (size_t)H * 256 + n_raw * values_raw_stage(vblk_bytes) + 1024;
}

// Grid of the value kernel: one CTA per SM, more when a CTA would hold more
// than kMaxRuns sequences or kMaxTiles tiles.  *slots = the most runs one CTA
// can hold.
static int values_grid(long long U, int n_st, int* slots) {
  long long G = std::min<long long>(num_sms(), U);
  for (;;) {
    const long long per = (U + G - 1) / G;
    const int sl = (int)((per + n_st - 1) / n_st) + 1;
    if ((sl <= kMaxRuns && per <= kMaxTiles / 2) || G >= U) {
      *slots = sl;
      return (int)G;
    }
    G = std::min(U, G * 2);
  }
}

bool plan_values_tc(starkv_layer* L) {
  const LayerView& v = L->view;
  const starkv_layer_config& c = L->cfg;
  if (!L->tc_scores) return false;
  // power-of-two count of 128-channel value blocks (at most two per team),
  // heads a multiple of 16; TMEM holds Y^T (nblk * H columns) and each team's
  // ring of at least two pages of A tiles (8 columns per block)
  if (v.rv % 128 != 0 || ((v.rv / 128) & (v.rv / 128 - 1)) != 0 || v.H % 16 != 0 || v.H > 64) return false;
  const int nblk = v.rv / 128;
  if (nblk > 2 * kTeams) return false;
  const int nbt = nblk > kTeams ? 2 : 1, n_teams = std::min(kTeams, nblk);
  L->val_na = std::min(kMaxASlots, (512 - nblk * v.H) / (n_teams * nbt * 16));   // slots of two pages
  if (L->val_na < 2) return false;
  const LatentDesc& ld = L->lat[v.L - 1];
  if (!ld.cmajor) return false;
  size_t bytes = 0;
  if (v.quantized) {
    if (ld.n_groups * 32 != v.rv) return false;
    for (int g = 0; g < ld.n_groups; ++g) {
      const GroupDesc& gd = L->grp[ld.group0 + g];
      if (gd.n != 32 || (gd.bits != 3 && gd.bits != 4) || gd.start != g * 32) return false;
    }
    // bytes of the value block: scales + code blocks
    bytes = ld.scale_bytes;
    for (int g = 0; g < ld.n_groups; ++g) bytes += (size_t)kPage * 32 * L->grp[ld.group0 + g].bits / 8;
  } else {
    if (c.dtype != STARKV_BF16 || ld.n_groups != 1) return false;
    bytes = (size_t)kPage * v.rv * 2;   // [channel][slot] bf16
  }
  L->val_bf16 = !v.quantized;
  L->vblk_off = ld.block_off;
  L->vblk_bytes = (int)bytes;
  // as many raw stages as fit next to the static tables and barriers
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, k_values_tc<2, false>) != cudaSuccess) return false;
  const int min_raw = 4;
  L->val_raw = 0;
  for (int n_raw = kMaxRawStages; n_raw >= min_raw && !L->val_raw; --n_raw)
    if (values_smem(v.H, L->vblk_bytes, n_raw) + fa.sharedSizeBytes <= 232448) L->val_raw = n_raw;
  return L->val_raw > 0;
}

size_t values_tc_ws_bytes(const starkv_layer* L, int batch, int max_len) {
  const int n_st = (max_len + kVSuper - 1) / kVSuper;
  const long long U = (long long)batch * n_st;
  int slots = 0;
  const int G = values_grid(U, n_st, &slots);
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  const LayerView& v = L->view;
  return r(sizeof(float) * (size_t)G * slots * v.H * v.rv) + 2 * r(sizeof(float) * (size_t)G * slots * v.H);
}

cudaError_t launch_values_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const ScoreOut& so, void* ws,
                             void* ytiles, cudaStream_t s, cudaEvent_t ev_mid) {
  const LayerView& v = L->view;
  const int max_len = max_pages * kPage;
  const int n_st = (max_len + kVSuper - 1) / kVSuper;
  const long long U = (long long)batch * n_st;
  int slots = 0;
  const int G = values_grid(U, n_st, &slots);
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
  a.raw_stage = (int)values_raw_stage(L->vblk_bytes);
  a.n_raw = L->val_raw;
  a.na = L->val_na;
  a.vgrp = L->d_grp + L->lat[v.L - 1].group0;
  a.rv = v.rv;
  a.H = v.H;
  a.lg_nblk = 0;
  while ((128 << a.lg_nblk) < v.rv) ++a.lg_nblk;
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
  a.status = L->status;
  const size_t smem = values_smem(v.H, L->vblk_bytes, L->val_raw);
  const bool two = v.rv / 128 > kTeams;   // two channel blocks per team
  const bool bf = L->val_bf16;
  const void* kern = two ? (bf ? (const void*)k_values_tc<2, true> : (const void*)k_values_tc<2, false>)
                         : (bf ? (const void*)k_values_tc<1, true> : (const void*)k_values_tc<1, false>);
  cudaError_t e = set_smem_limit(kern, smem);
  if (e != cudaSuccess) return e;
  if (two && bf)
    k_values_tc<2, true><<<G, kValThreads, smem, s>>>(a);
  else if (two)
    k_values_tc<2, false><<<G, kValThreads, smem, s>>>(a);
  else if (bf)
    k_values_tc<1, true><<<G, kValThreads, smem, s>>>(a);
  else
    k_values_tc<1, false><<<G, kValThreads, smem, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
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
                             void* out, void* ws, size_t ws_bytes, cudaStream_t s, bool profile) {
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
  // optional timing events between the kernels (see starkv_profile_decode)
  cudaEvent_t* ev = nullptr;
  if (profile && L->prof_n > 0) {
    starkv_layer* Lm = const_cast<starkv_layer*>(L);
    const int slot = (int)(Lm->prof_calls++ % Lm->prof_n);
    ev = &Lm->prof_ev[(size_t)slot * (STARKV_N_PHASES + 1)];
    Lm->prof_used[slot] = 1;
  }
  cudaError_t e;
  if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return e;
  ScoreOut so;
  e = launch_scores_tc(L, pool, n_pages, pt, max_pages, batch, seq_lens, q_pos, q, w_scores, &so, nullptr, 0, s);
  if (e != cudaSuccess) return e;
  if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return e;
  if (batch % NB != 0 || L->Kp != L->view.H * L->view.wv) {
    e = cudaMemsetAsync(ytiles, 0, y_bytes, s);
    if (e != cudaSuccess) return e;
  }
  e = launch_values_tc(L, pool, n_pages, pt, max_pages, batch, seq_lens, so, w_values, ytiles, s, ev ? ev[2] : nullptr);
  if (e != cudaSuccess) return e;
  if (ev && (e = cudaEventRecord(ev[3], s)) != cudaSuccess) return e;
  e = launch_outproj_tc(L, ytiles, batch, out, part, s);
  if (e != cudaSuccess) return e;
  if (ev && (e = cudaEventRecord(ev[4], s)) != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace starkv
