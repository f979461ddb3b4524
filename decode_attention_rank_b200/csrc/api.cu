// Host side of the C ABI: argument checks, layer planning (page layout, group
// tables), factor folding at load time, and kernel dispatch.
#include <limits.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <string>

#include "starkv_internal.cuh"

namespace starkv {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

static size_t ru(size_t x, size_t m) { return (x + m - 1) / m * m; }

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = std::min(n, 256);   // persistent grids: one CTA per SM, at most 256
  }
  return cached[dev];
}

cudaError_t set_smem_limit(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[{kernel, dev}];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

// Channels of the high-precision segment: ceil(top_fraction * r) (reading notes
// "STAR-KV 阅读笔记" section 6.1; the model card's top_fraction).  The fraction
// arrives as a float: a product within its rounding error (r * 2^-23) of an
// integer is that integer, so that e.g. 0.2 (stored as 0.2000000030) gives 8
// channels of 40, not 9.
static int n_high(int r, float top_fraction) {
  return (int)ceil((double)top_fraction * (double)r - (double)r * 0x1p-23 - 1e-9);
}

}  // namespace starkv

using namespace starkv;

#define CHECK_ARG(cond, msg)            \
  do {                                  \
    if (!(cond)) {                      \
      set_error(msg);                   \
      return STARKV_ERR_ARG;            \
    }                                   \
  } while (0)

// Buffers that kernels reach with 16-byte accesses or bulk copies (pool, q,
// out, input, workspace) must start on a 16-byte boundary, int32 arrays on a
// 4-byte one; a misaligned pointer is refused on the host before any launch.
static bool aligned_to(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

#define CUDA_TRY(expr)                                                          \
  do {                                                                          \
    cudaError_t e_ = (expr);                                                    \
    if (e_ != cudaSuccess) {                                                    \
      set_error(std::string(#expr) + ": " + cudaGetErrorString(e_));           \
      return STARKV_ERR_CUDA;                                                   \
    }                                                                           \
  } while (0)

// Plan the page layout: latent blocks in order (keys per KV head, then values),
// each a multiple of 16 bytes; a quantized block is the scale block
// [group][slot] fp16 followed by one LSB-first code block per group.
static starkv_status plan_layer(starkv_layer* L) {
  const starkv_layer_config& c = L->cfg;
  const int Hkv = c.n_kv_heads, d = c.head_dim;
  const int es = c.dtype == STARKV_F32 ? 4 : 2;
  std::vector<int> widths;
  if (c.plain) {
    for (int h = 0; h < Hkv; ++h) widths.push_back(d);
    widths.push_back(Hkv * d);
  } else {
    for (int h = 0; h < Hkv; ++h) widths.push_back(L->key_ranks[h]);
    widths.push_back(c.value_rank);
  }
  const bool quant = c.quantized && !c.plain;
  size_t off = 0;
  int ch = 0;
  double bpt = 0;
  L->lat.clear();
  L->grp.clear();
  for (size_t li = 0; li < widths.size(); ++li) {
    LatentDesc ld{};
    ld.width = widths[li];
    ld.block_off = (int)off;
    ld.ch_off = ch;
    ld.group0 = (int)L->grp.size();
    ld.cmajor = (!c.plain && li + 1 == widths.size()) ? 1 : 0;
    if (!quant) {
      L->grp.push_back(GroupDesc{0, ld.width, 0, 0});
      ld.n_groups = 1;
      ld.scale_bytes = 0;
      off += ru((size_t)kPage * ld.width * es, 16);
      bpt += (double)ld.width * es;
    } else {
      const int nh = n_high(ld.width, c.top_fraction);
      const int seg_start[2] = {0, nh}, seg_len[2] = {nh, ld.width - nh}, seg_bits[2] = {c.top_bits, c.bottom_bits};
      std::vector<GroupDesc> gs;
      for (int s = 0; s < 2; ++s)
        for (int k = 0; k < seg_len[s]; k += c.group_size)
          gs.push_back(GroupDesc{seg_start[s] + k, std::min(c.group_size, seg_len[s] - k), seg_bits[s], 0});
      ld.n_groups = (int)gs.size();
      ld.n_hi = nh;
      ld.gsize = c.group_size;
      ld.scale_bytes = (int)ru((size_t)gs.size() * kPage * 2, 16);
      size_t boff = ld.scale_bytes;
      for (auto& g : gs) {
        g.code_off = (int)boff;
        boff += ru((size_t)kPage * g.n * g.bits / 8, 16);
        bpt += g.n * g.bits / 8.0 + 2.0;
      }
      for (auto& g : gs) L->grp.push_back(g);
      off += boff;
    }
    ch += ld.width;
    L->lat.push_back(ld);
  }
  L->page_bytes = ru(off, 128);
  L->bytes_per_token = bpt;
  LayerView& v = L->view;
  v.D = c.hidden;
  v.H = c.n_heads;
  v.Hkv = Hkv;
  v.d = d;
  v.group_q = c.n_heads / Hkv;
  v.L = (int)widths.size();
  v.Ltot = ch;
  v.Rk = ch - widths.back();
  v.rv = widths.back();
  v.wv = c.plain ? d : c.value_rank;
  v.es = es;
  v.dtype = c.dtype;
  v.quantized = quant ? 1 : 0;
  v.plain = c.plain ? 1 : 0;
  v.rope = c.rope ? 1 : 0;
  v.hadamard = (quant && c.hadamard_block) ? 1 : 0;
  v.rope_log2_theta = (float)log2(c.rope_theta);
  const float sc = c.softmax_scale > 0 ? c.softmax_scale : (float)(1.0 / sqrt((double)d));
  v.scale_log2 = sc * kLog2e;
  v.page_bytes = (long long)L->page_bytes;
  L->Kp = (int)ru((size_t)c.n_heads * v.wv, 64);
  L->Dp = (int)ru((size_t)c.hidden, 128);
  L->key_off.assign(Hkv + 1, 0);
  for (int h = 0; h < Hkv; ++h) L->key_off[h + 1] = L->key_off[h] + widths[h];
  const size_t mel = c.dtype == STARKV_F32 ? 4 : 2;
  L->unfused = c.unfused_output ? 1 : 0;
  L->factor_bytes = (c.plain ? 0 : (size_t)v.Rk * d * (c.dtype == STARKV_F32 ? 4 : 2)) +
                    (L->unfused ? 2 * (size_t)c.n_heads * d * ((size_t)v.rv + c.hidden)   // B'_v per head + W_o
                                : (size_t)c.hidden * c.n_heads * v.wv * mel);             // M
  return STARKV_OK;
}

static starkv_status check_config(const starkv_layer_config* c) {
  CHECK_ARG(c != nullptr, "config is NULL");
  CHECK_ARG(c->hidden > 0 && c->n_heads > 0 && c->n_kv_heads > 0 && c->head_dim > 0, "non-positive shape");
  CHECK_ARG(c->n_heads % c->n_kv_heads == 0, "n_heads must be a multiple of n_kv_heads");
  CHECK_ARG(c->head_dim % 2 == 0 && c->head_dim <= 256, "head_dim must be even and <= 256");
  CHECK_ARG(c->dtype == STARKV_F32 || c->dtype == STARKV_BF16, "dtype must be STARKV_F32 or STARKV_BF16");
  CHECK_ARG(c->page_size == 16, "page_size must be 16");
  CHECK_ARG(c->n_heads <= 128, "n_heads must be <= 128");
  if (!c->plain) {
    CHECK_ARG(c->key_ranks != nullptr, "key_ranks is NULL");
    for (int h = 0; h < c->n_kv_heads; ++h)
      CHECK_ARG(c->key_ranks[h] >= 1 && c->key_ranks[h] <= c->head_dim, "key rank outside 1..head_dim");
    CHECK_ARG(c->value_rank >= 1 && c->value_rank <= c->n_kv_heads * c->head_dim, "value_rank outside 1..H_kv*d");
  }
  if (c->quantized && !c->plain) {
    CHECK_ARG(c->top_bits >= 2 && c->top_bits <= 8 && c->bottom_bits >= 2 && c->bottom_bits <= 8,
              "code widths must be 2..8 bits");
    CHECK_ARG(c->group_size >= 1 && c->group_size <= 32, "group_size must be 1..32");
    CHECK_ARG(c->top_fraction >= 0.f && c->top_fraction <= 1.f, "top_fraction must be in [0, 1]");
  }
  if (c->hadamard_block) {
    CHECK_ARG(c->quantized && !c->plain, "hadamard_block requires a quantized compressed layer");
    CHECK_ARG(c->hadamard_block == c->group_size, "hadamard_block must equal group_size");
  }
  if (c->rope) CHECK_ARG(c->rope_theta > 1.0, "rope_theta must be > 1");
  if (c->unfused_output) {
    CHECK_ARG(c->dtype == STARKV_BF16 && !c->plain && c->head_dim == 128 && c->value_rank % 64 == 0,
              "unfused_output needs a bf16 compressed layer with head_dim 128 and value_rank a multiple of 64");
  }
  return STARKV_OK;
}

extern "C" {

const char* starkv_status_string(starkv_status s) {
  switch (s) {
    case STARKV_OK: return "ok";
    case STARKV_ERR_ARG: return "invalid argument";
    case STARKV_ERR_UNSUPPORTED: return "unsupported";
    case STARKV_ERR_OOM: return "out of device memory";
    case STARKV_ERR_CUDA: return "CUDA error";
    case STARKV_ERR_DEVICE: return "device status word set";
    case STARKV_ERR_TIMEOUT: return "device wait timed out";
    case STARKV_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* starkv_last_error(void) { return g_last_error.c_str(); }

const char* starkv_version(void) { return "starkv-b200 0.1 (sm_100a)"; }

void starkv_free_layer(starkv_layer* L) {
  if (!L) return;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(L->device);
  cudaFree(L->d_lat);
  cudaFree(L->d_grp);
  cudaFree(L->d_key_off);
  cudaFree(L->d_grp_lat);
  cudaFree(L->A_T);
  cudaFree(L->A_tiles);
  cudaFree(L->Bk);
  cudaFree(L->M_T);
  cudaFree(L->Bv_tiles);
  cudaFree(L->Bk_tiles);
  cudaFree(L->Wo_tiles);
  cudaFree(L->status);
  cudaFree(L->d_items);
  cudaFree(L->d_score_heads);
  cudaFree(L->rope_E);
  for (cudaEvent_t e : L->prof_ev) cudaEventDestroy(e);
  cudaSetDevice(cur);
  delete L;
}

starkv_status starkv_load_factors(const starkv_layer_config* cfg, const void* A_k, const void* B_k, const void* A_v,
                                  const void* B_v, const void* W_o, starkv_stream_t stream, starkv_layer** out) {
  set_error("");
  CHECK_ARG(out != nullptr, "out is NULL");
  *out = nullptr;
  starkv_status st = check_config(cfg);
  if (st != STARKV_OK) return st;
  CHECK_ARG(A_k && A_v && W_o, "A_k, A_v and W_o must be non-NULL");
  if (!cfg->plain) CHECK_ARG(B_k && B_v, "B_k and B_v must be non-NULL");
  cudaStream_t s = (cudaStream_t)stream;
  starkv_layer* L = new starkv_layer();
  L->cfg = *cfg;
  if (!cfg->plain) L->key_ranks.assign(cfg->key_ranks, cfg->key_ranks + cfg->n_kv_heads);
  L->cfg.key_ranks = nullptr;
  cudaGetDevice(&L->device);
  plan_layer(L);
  LayerView& v = L->view;
  const int D = v.D, d = v.d, H = v.H;
  const size_t es = cfg->dtype == STARKV_F32 ? 4 : 2;
  auto fail = [&](starkv_status code, const char* what) {
    set_error(std::string("load_factors: ") + what + ": " + cudaGetErrorString(cudaGetLastError()));
    starkv_free_layer(L);
    return code;
  };
  if (cudaMalloc(&L->d_lat, sizeof(LatentDesc) * L->lat.size()) != cudaSuccess ||
      cudaMalloc(&L->d_grp, sizeof(GroupDesc) * L->grp.size()) != cudaSuccess ||
      cudaMalloc(&L->d_key_off, sizeof(int) * L->key_off.size()) != cudaSuccess ||
      cudaMalloc(&L->status, sizeof(uint32_t)) != cudaSuccess ||
      cudaMalloc(&L->A_T, es * (size_t)v.Ltot * D) != cudaSuccess)
    return fail(STARKV_ERR_OOM, "cudaMalloc");
  const size_t wo_tiles_bytes = (size_t)(L->Dp / 128) * (H * d / 64) * 16384;
  // B'_v per head and W_o as tiles: the unfused output's factors, and the
  // prefill's value reconstruction and output (bf16 compressed layers)
  const bool bv_wo = L->unfused || (cfg->dtype == STARKV_BF16 && !cfg->plain && d == 128 && v.rv % 64 == 0);
  if (bv_wo && (cudaMalloc(&L->Bv_tiles, (size_t)H * (v.rv / 64) * 16384) != cudaSuccess ||
                cudaMalloc(&L->Wo_tiles, wo_tiles_bytes) != cudaSuccess))
    return fail(STARKV_ERR_OOM, "cudaMalloc");
  if (!L->unfused &&
      cudaMalloc(&L->M_T, cfg->dtype == STARKV_F32 ? 4 * (size_t)D * H * v.wv : 2 * (size_t)L->Dp * L->Kp) != cudaSuccess)
    return fail(STARKV_ERR_OOM, "cudaMalloc");
  if (!cfg->plain && cudaMalloc(&L->Bk, sizeof(float) * (size_t)v.Rk * d) != cudaSuccess)
    return fail(STARKV_ERR_OOM, "cudaMalloc");
  v.lat = L->d_lat;
  v.grp = L->d_grp;
  v.status = L->status;
  std::vector<int> grp_lat(L->grp.size());
  for (size_t li = 0; li < L->lat.size(); ++li)
    for (int g = 0; g < L->lat[li].n_groups; ++g) grp_lat[L->lat[li].group0 + g] = (int)li;
  if (cudaMalloc(&L->d_grp_lat, sizeof(int) * grp_lat.size()) != cudaSuccess) return fail(STARKV_ERR_OOM, "cudaMalloc");
  if (cudaMemcpy(L->d_grp_lat, grp_lat.data(), sizeof(int) * grp_lat.size(), cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(STARKV_ERR_CUDA, "upload group table");
  if (cudaMemcpyAsync(L->d_lat, L->lat.data(), sizeof(LatentDesc) * L->lat.size(), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(L->d_grp, L->grp.data(), sizeof(GroupDesc) * L->grp.size(), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(L->d_key_off, L->key_off.data(), sizeof(int) * L->key_off.size(), cudaMemcpyHostToDevice, s) ||
      cudaMemsetAsync(L->status, 0, sizeof(uint32_t), s) ||
      (L->M_T && cfg->dtype != STARKV_F32 && cudaMemsetAsync(L->M_T, 0, 2 * (size_t)L->Dp * L->Kp, s)) ||
      (L->Wo_tiles && cudaMemsetAsync(L->Wo_tiles, 0, wo_tiles_bytes, s)))
    return fail(STARKV_ERR_CUDA, "upload tables");
  // Projection rows A_T[ch][k] for every latent channel (keys, then values).
  if (cfg->plain) {
    if (launch_transpose_into(A_k, D, v.Rk, cfg->dtype, L->A_T, 0, D, s) ||
        launch_transpose_into(A_v, D, v.rv, cfg->dtype, L->A_T, v.Rk, D, s))
      return fail(STARKV_ERR_CUDA, "transpose W_k/W_v");
  } else {
    size_t elem_off = 0;
    for (int h = 0; h < v.Hkv; ++h) {
      const char* src = (const char*)A_k + elem_off * es;
      if (launch_transpose_into(src, D, L->key_ranks[h], cfg->dtype, L->A_T, L->key_off[h], D, s))
        return fail(STARKV_ERR_CUDA, "transpose A_k");
      elem_off += (size_t)D * L->key_ranks[h];
    }
    if (launch_transpose_into(A_v, D, v.rv, cfg->dtype, L->A_T, v.Rk, D, s))
      return fail(STARKV_ERR_CUDA, "transpose A_v");
    // B'_k = R^T B_k per KV head (float32).
    size_t boff = 0;
    for (int h = 0; h < v.Hkv; ++h) {
      const char* src = (const char*)B_k + boff * es;
      if (launch_rotate_rows(L, src, cfg->dtype, h, d, L->Bk + (size_t)L->key_off[h] * d, s))
        return fail(STARKV_ERR_CUDA, "rotate B_k");
      boff += (size_t)L->key_ranks[h] * d;
    }
  }
  // the projection rows again as fp16 128 x 64 tiles for the tensor-core projection
  if (cfg->dtype == STARKV_BF16) {
    const size_t tb = (size_t)((v.Ltot + 127) / 128) * ((D + 63) / 64) * 16384;
    if (cudaMalloc(&L->A_tiles, tb) != cudaSuccess) return fail(STARKV_ERR_OOM, "cudaMalloc");
    if (launch_pack_rows_tiles(L->A_T, v.Ltot, D, L->A_tiles, s, 128) != cudaSuccess)
      return fail(STARKV_ERR_CUDA, "tile A");
  }
  // M_h = B'_v,kv(h) W_o,h, stored transposed as M_T [D][H * wv].
  float* Bv_rot = nullptr;
  if (!cfg->plain) {
    if (cudaMalloc(&Bv_rot, sizeof(float) * (size_t)v.rv * v.Hkv * d) != cudaSuccess)
      return fail(STARKV_ERR_OOM, "cudaMalloc");
    if (launch_rotate_rows(L, B_v, cfg->dtype, v.Hkv, v.Hkv * d, Bv_rot, s)) {
      cudaFree(Bv_rot);
      return fail(STARKV_ERR_CUDA, "rotate B_v");
    }
  }
  cudaError_t e = L->unfused ? launch_build_unfused(L, Bv_rot, W_o, s) : launch_fold_M(L, Bv_rot, W_o, s);
  if (e == cudaSuccess && !L->unfused && L->Bv_tiles) e = launch_build_unfused(L, Bv_rot, W_o, s);
  // B'_k as tiles for the prefill's key rebuild (key ranks up to 64)
  if (e == cudaSuccess && L->Bv_tiles && *std::max_element(L->key_ranks.begin(), L->key_ranks.end()) <= 64) {
    if (cudaMalloc(&L->Bk_tiles, (size_t)v.Hkv * 16384) != cudaSuccess) {
      if (Bv_rot) cudaFree(Bv_rot);
      return fail(STARKV_ERR_OOM, "cudaMalloc");
    }
    e = launch_prefill_bk_tiles(L, L->Bk_tiles, s);
  }
  if (Bv_rot) {
    cudaStreamSynchronize(s);
    cudaFree(Bv_rot);
  }
  if (e != cudaSuccess) return fail(STARKV_ERR_CUDA, "fold M");
  // tensor-core score kernel: MMA items, RoPE table
  L->tc_scores = plan_scores_tc(L);
  L->tc_values = L->tc_scores && plan_values_tc(L);
  if (L->tc_scores) {
    if (cudaMalloc(&L->d_items, sizeof(ScoreItem) * L->items.size()) != cudaSuccess ||
        cudaMalloc(&L->d_score_heads, sizeof(ScoreHead) * L->score_heads.size()) != cudaSuccess ||
        cudaMalloc(&L->rope_E, (size_t)L->rope_tiles * 32768) != cudaSuccess)
      return fail(STARKV_ERR_OOM, "cudaMalloc");
    if (cudaMemcpyAsync(L->d_items, L->items.data(), sizeof(ScoreItem) * L->items.size(), cudaMemcpyHostToDevice,
                        s) != cudaSuccess ||
        cudaMemcpyAsync(L->d_score_heads, L->score_heads.data(), sizeof(ScoreHead) * L->score_heads.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess ||
        build_rope_table(L, s) != cudaSuccess)
      return fail(STARKV_ERR_CUDA, "rope table");
    cudaStreamSynchronize(s);   // the item tables live in host vectors that must outlive the copies
  }
  *out = L;
  return STARKV_OK;
}

starkv_status starkv_layer_get_info(const starkv_layer* L, starkv_layer_info* info) {
  CHECK_ARG(L && info, "NULL argument");
  info->n_latents = L->view.L;
  info->latent_total = L->view.Ltot;
  info->key_rank_total = L->view.Rk;
  info->page_bytes = L->page_bytes;
  info->bytes_per_token = L->bytes_per_token;
  info->factor_bytes = L->factor_bytes;
  return STARKV_OK;
}

size_t starkv_page_bytes(const starkv_layer* L) { return L ? L->page_bytes : 0; }

starkv_status starkv_cache_init(const starkv_layer* L, void* pool, int64_t n_pages, starkv_stream_t stream) {
  set_error("");
  CHECK_ARG(L && pool, "NULL argument");
  CHECK_ARG(n_pages >= 0, "negative n_pages");
  CHECK_ARG(((uintptr_t)pool & 15) == 0, "pool must be 16-byte aligned");
  CUDA_TRY(cudaMemsetAsync(pool, 0, (size_t)n_pages * L->page_bytes, (cudaStream_t)stream));
  return STARKV_OK;
}

size_t starkv_append_workspace_bytes(const starkv_layer* L, int n_tokens) {
  if (!L || n_tokens <= 0) return 0;
  size_t b = ru(sizeof(float) * (size_t)n_tokens * L->view.Ltot, 256);
  if (L->A_tiles)
    b += ru(rows_tiles_bytes(n_tokens, L->view.D), 256) + ru(gemm_part_bytes(L->view.Ltot, L->view.D, n_tokens), 256);
  return b;
}

starkv_status starkv_append(const starkv_layer* L, void* pool, int64_t n_pages, const int32_t* page_table,
                            int n_seqs, int max_pages, int n_tokens, const int32_t* seq_idx, const int32_t* positions,
                            const void* input, int input_is_latent, void* workspace, size_t ws_bytes,
                            starkv_stream_t stream) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(n_tokens >= 0, "negative n_tokens");
  if (n_tokens == 0) return STARKV_OK;
  CHECK_ARG(pool && page_table && seq_idx && positions && input, "NULL buffer");
  CHECK_ARG(((uintptr_t)pool & 15) == 0, "pool must be 16-byte aligned");
  CHECK_ARG(n_pages > 0 && max_pages > 0 && n_seqs > 0, "empty pool or page table");
  CHECK_ARG(max_pages <= INT_MAX / kPage, "max_pages * 16 overflows int");
  CHECK_ARG(aligned_to(page_table, 4) && aligned_to(seq_idx, 4) && aligned_to(positions, 4),
            "page_table, seq_idx and positions must be 4-byte aligned");
  CHECK_ARG(aligned_to(input, 16) && aligned_to(workspace, 16), "input and workspace must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  const float* z = (const float*)input;
  if (!input_is_latent) {
    const size_t need = starkv_append_workspace_bytes(L, n_tokens);
    if (ws_bytes < need || workspace == nullptr) {
      set_error("append workspace too small");
      return STARKV_ERR_WORKSPACE;
    }
    if (L->A_tiles) {
      // tensor cores: z^T = A_T x^T with the stream-K GEMM of the output projection
      uint8_t* w = (uint8_t*)workspace;
      float* zw = (float*)w;
      w += ru(sizeof(float) * (size_t)n_tokens * L->view.Ltot, 256);
      void* xt = w;
      w += ru(rows_tiles_bytes(n_tokens, L->view.D), 256);
      CUDA_TRY(launch_pack_rows_tiles(input, n_tokens, L->view.D, xt, s));
      CUDA_TRY(launch_gemm_tc((const uint8_t*)L->A_tiles, L->view.Ltot, L->view.D, L->view.Ltot, xt, n_tokens, zw,
                              true, (float*)w, L->status, s));
    } else {
      CUDA_TRY(launch_project(L, input, n_tokens, (float*)workspace, s));
    }
    z = (const float*)workspace;
  }
  const int rotate = (!input_is_latent && L->view.hadamard) ? 1 : 0;
  const int rope_keys = (!input_is_latent && L->view.plain && L->view.rope) ? 1 : 0;
  CUDA_TRY(launch_pack(L, (uint8_t*)pool, n_pages, page_table, n_seqs, max_pages, n_tokens, seq_idx, positions, z,
                       rotate, rope_keys, s));
  return STARKV_OK;
}

namespace starkv {
namespace {

// Prefill rows go through the tensor-core decode kernels in batches of at most
// this many query rows (the output GEMM's widest B tile).
constexpr int kPrefillRows = 256;

// Page-table rows of query rows: out[r][p] = page_table[seq[r]][p].
__global__ void k_expand_rows(const int32_t* __restrict__ page_table, int max_pages, const int32_t* __restrict__ seq,
                              int rows, int32_t* __restrict__ out) {
  const long long n = (long long)rows * max_pages;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / max_pages), p = (int)(i % max_pages);
    out[i] = page_table[(size_t)seq[r] * max_pages + p];
  }
}

// Workspace of a tensor-core prefill: the row table, one batch of expanded
// page-table rows and one batch's decode workspace.
size_t prefill_tc_ws_bytes(const starkv_layer* L, long long rows, int max_pages) {
  const int nb = (int)std::min<long long>(rows, kPrefillRows);
  return ru(sizeof(int32_t) * 3 * (size_t)rows, 256) + ru(sizeof(int32_t) * (size_t)nb * max_pages, 256) +
         decode_tc_ws_bytes(L, nb, max_pages * kPage);
}

}  // namespace
}  // namespace starkv

size_t starkv_workspace_bytes(const starkv_layer* L, int batch, int max_ctx, int max_q) {
  if (!L || batch <= 0) return 0;
  if (max_q < 1) max_q = 1;
  max_ctx = std::max(max_ctx, 1);
  size_t need = decode_generic_ws_bytes(L, batch, max_ctx, false);
  if (L->tc_scores) need += scores_tc_ws_bytes(L, batch, max_ctx);
  if (L->tc_values) need = std::max(need, decode_tc_ws_bytes(L, batch, max_ctx));
  if (max_q > 1) {
    const long long rows = std::min<long long>((long long)batch * max_q, 1 << 30);
    need = std::max(need, ru(sizeof(int32_t) * 3 * (size_t)rows, 256) +
                              decode_generic_ws_bytes(L, (int)rows, max_ctx, true));
    if (L->tc_scores && L->tc_values)
      need = std::max(need, prefill_tc_ws_bytes(L, rows, (max_ctx + kPage - 1) / kPage));
    if (prefill_flash_supported(L)) need = std::max(need, prefill_flash_ws_bytes(L, max_ctx, max_q));
  }
  return need;
}

starkv_status starkv_decode_attn(const starkv_layer* L, const void* pool, int64_t n_pages, const int32_t* page_table,
                                 int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos,
                                 const void* q, void* out, void* workspace, size_t ws_bytes, starkv_stream_t stream) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(batch >= 0, "negative batch");
  if (batch == 0) return STARKV_OK;
  CHECK_ARG(pool && page_table && seq_lens && q && out, "NULL buffer");
  CHECK_ARG(n_pages > 0 && max_pages > 0, "empty pool or page table");
  CHECK_ARG(max_pages <= INT_MAX / kPage, "max_pages * 16 overflows int");
  CHECK_ARG(aligned_to(pool, 16) && aligned_to(q, 16) && aligned_to(out, 16) && aligned_to(workspace, 16),
            "pool, q, out and workspace must be 16-byte aligned");
  CHECK_ARG(aligned_to(page_table, 4) && aligned_to(seq_lens, 4) && aligned_to(q_pos, 4),
            "page_table, seq_lens and q_pos must be 4-byte aligned");
  const int max_len = max_pages * kPage;
  const bool tc_ok = L->tc_scores && max_len <= L->rope_tiles * 128;
  const bool use_tc_all = tc_ok && L->tc_values && L->decode_path == 0;
  const bool use_tc_scores = tc_ok && (L->decode_path == 2 || L->decode_path == 0);
  size_t need = decode_generic_ws_bytes(L, batch, max_len, false) +
                (L->tc_scores ? scores_tc_ws_bytes(L, batch, max_len) : 0);
  if (use_tc_all) need = decode_tc_ws_bytes(L, batch, max_len);
  if (workspace == nullptr || ws_bytes < need) {
    set_error("decode workspace too small: need " + std::to_string(need) + " bytes");
    return STARKV_ERR_WORKSPACE;
  }
  if (use_tc_all) {
    CUDA_TRY(launch_decode_tc(L, (const uint8_t*)pool, n_pages, page_table, max_pages, batch, seq_lens, q_pos, q, out,
                              workspace, ws_bytes, (cudaStream_t)stream));
    return STARKV_OK;
  }
  RowInfo ri{nullptr, seq_lens, q_pos};
  CUDA_TRY(launch_decode_generic(L, (const uint8_t*)pool, n_pages, page_table, max_pages, batch, ri, max_len, q, out,
                                 workspace, ws_bytes, false, (cudaStream_t)stream, use_tc_scores));
  return STARKV_OK;
}

starkv_status starkv_prefill_attn(const starkv_layer* L, const void* pool, int64_t n_pages, const int32_t* page_table,
                                  int max_pages, int batch, const int32_t* q_start_host, const int32_t* q_len_host,
                                  const void* q, void* out, void* workspace, size_t ws_bytes, starkv_stream_t stream) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(batch >= 0, "negative batch");
  if (batch == 0) return STARKV_OK;
  CHECK_ARG(pool && page_table && q_start_host && q_len_host && q && out, "NULL buffer");
  CHECK_ARG(n_pages > 0 && max_pages > 0, "empty pool or page table");
  CHECK_ARG(max_pages <= INT_MAX / kPage, "max_pages * 16 overflows int");
  CHECK_ARG(aligned_to(pool, 16) && aligned_to(q, 16) && aligned_to(out, 16) && aligned_to(workspace, 16),
            "pool, q, out and workspace must be 16-byte aligned");
  CHECK_ARG(aligned_to(page_table, 4), "page_table must be 4-byte aligned");
  std::vector<int32_t> tab;
  int rows = 0, max_len = 0;
  for (int b = 0; b < batch; ++b) {
    CHECK_ARG(q_start_host[b] >= 0 && q_len_host[b] >= 0, "negative q_start or q_len");
    CHECK_ARG((long long)q_start_host[b] + q_len_host[b] <= (long long)max_pages * kPage,
              "queries beyond the page table");
    rows += q_len_host[b];
    max_len = std::max(max_len, q_start_host[b] + q_len_host[b]);
  }
  if (rows == 0) return STARKV_OK;
  cudaStream_t s = (cudaStream_t)stream;
  // Tensor-core prefill: per sequence, keys and values rebuilt once for the
  // chunk, then tiled causal attention and the output through W_o.
  {
    int max_q = 0;
    for (int b = 0; b < batch; ++b) max_q = std::max(max_q, q_len_host[b]);
    const bool flash = prefill_flash_supported(L) && L->decode_path == 0 &&
                       (L->view.plain || max_len <= L->rope_tiles * 128) && workspace != nullptr &&
                       ws_bytes >= prefill_flash_ws_bytes(L, max_len, max_q);
    if (flash) {
      const size_t qrow = (size_t)L->view.H * L->cfg.head_dim * sizeof(uint16_t);
      const size_t orow = (size_t)L->view.D * (L->cfg.dtype == STARKV_F32 ? 4 : 2);
      long long r0 = 0;
      for (int b = 0; b < batch; ++b) {
        CUDA_TRY(launch_prefill_flash(L, (const uint8_t*)pool, n_pages, page_table + (size_t)b * max_pages,
                                      q_start_host[b], q_len_host[b], (const char*)q + r0 * qrow,
                                      (char*)out + r0 * orow, workspace, max_len, max_q, s));
        r0 += q_len_host[b];
      }
      return STARKV_OK;
    }
  }
  tab.resize(3 * (size_t)rows);
  int r = 0;
  for (int b = 0; b < batch; ++b)
    for (int i = 0; i < q_len_host[b]; ++i, ++r) {
      tab[r] = b;                                // sequence
      tab[rows + r] = q_start_host[b] + i + 1;   // visible length
      tab[2 * rows + r] = q_start_host[b] + i;   // RoPE position
    }
  const size_t tab_bytes = ru(sizeof(int32_t) * tab.size(), 256);
  int32_t* dtab = (int32_t*)workspace;
  // Tensor-core path: every query row is a decode of its sequence at its
  // visible length and RoPE position, run through the tensor-core decode
  // kernels in batches of kPrefillRows rows that share the workspace.
  // A workspace sized for a shorter context than the page table's capacity
  // (enough for the CUDA-core kernels) takes the CUDA-core path.
  const bool tc = L->tc_scores && L->tc_values && L->decode_path == 0 && max_pages * kPage <= L->rope_tiles * 128 &&
                  workspace != nullptr && ws_bytes >= prefill_tc_ws_bytes(L, rows, max_pages);
  if (tc) {
    const int nb = std::min(rows, kPrefillRows);
    int32_t* pt_rows = (int32_t*)((char*)workspace + tab_bytes);
    char* ws_tc = (char*)workspace + tab_bytes + ru(sizeof(int32_t) * (size_t)nb * max_pages, 256);
    const size_t ws_tc_bytes = ws_bytes - (size_t)(ws_tc - (char*)workspace);
    const size_t qrow = (size_t)L->view.H * L->cfg.head_dim * sizeof(uint16_t);
    const size_t orow = (size_t)L->view.D * sizeof(uint16_t);
    CUDA_TRY(cudaMemcpyAsync(dtab, tab.data(), sizeof(int32_t) * tab.size(), cudaMemcpyHostToDevice, s));
    for (int r0 = 0; r0 < rows; r0 += nb) {
      const int n = std::min(nb, rows - r0);
      k_expand_rows<<<std::max(1, std::min(1024, (int)(((long long)n * max_pages + 255) / 256))), 256, 0, s>>>(
          page_table, max_pages, dtab + r0, n, pt_rows);
      CUDA_TRY(cudaGetLastError());
      CUDA_TRY(launch_decode_tc(L, (const uint8_t*)pool, n_pages, pt_rows, max_pages, n, dtab + rows + r0,
                                dtab + 2 * rows + r0, (const char*)q + (size_t)r0 * qrow, (char*)out + (size_t)r0 * orow,
                                ws_tc, ws_tc_bytes, s, false));
    }
    // pageable host source: make sure the copy has consumed `tab` before it is freed
    CUDA_TRY(cudaStreamSynchronize(s));
    return STARKV_OK;
  }
  const size_t need = tab_bytes + decode_generic_ws_bytes(L, rows, max_len, true);
  if (workspace == nullptr || ws_bytes < need) {
    set_error("prefill workspace too small: need " + std::to_string(need) + " bytes");
    return STARKV_ERR_WORKSPACE;
  }
  CUDA_TRY(cudaMemcpyAsync(dtab, tab.data(), sizeof(int32_t) * tab.size(), cudaMemcpyHostToDevice, s));
  RowInfo ri{dtab, dtab + rows, dtab + 2 * rows};
  CUDA_TRY(launch_decode_generic(L, (const uint8_t*)pool, n_pages, page_table, max_pages, rows, ri, max_len, q, out,
                                 (char*)workspace + tab_bytes, ws_bytes - tab_bytes, true, s));
  // pageable host source: make sure the copy has consumed `tab` before it is freed
  CUDA_TRY(cudaStreamSynchronize(s));
  return STARKV_OK;
}

starkv_status starkv_set_decode_path(starkv_layer* L, int path) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(path >= 0 && path <= 2, "path must be 0, 1 or 2");
  if (path == 2 && !L->tc_scores) {
    set_error("this layer's shape does not fit the tensor-core score kernel");
    return STARKV_ERR_UNSUPPORTED;
  }
  L->decode_path = path;
  return STARKV_OK;
}

starkv_status starkv_profile_decode(starkv_layer* L, int n_calls) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(n_calls >= 0 && n_calls <= 4096, "n_calls must be in [0, 4096]");
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(L->device);
  for (cudaEvent_t e : L->prof_ev) cudaEventDestroy(e);
  L->prof_ev.clear();
  L->prof_used.assign(n_calls, 0);
  L->prof_n = 0;
  L->prof_calls = 0;
  for (int i = 0; i < n_calls * (STARKV_N_PHASES + 1); ++i) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaSetDevice(cur);
      set_error("cudaEventCreate failed");
      return STARKV_ERR_CUDA;
    }
    L->prof_ev.push_back(e);
  }
  L->prof_n = n_calls;
  cudaSetDevice(cur);
  return STARKV_OK;
}

starkv_status starkv_decode_phase_ms(const starkv_layer* L, float* ms, int n_calls) {
  set_error("");
  CHECK_ARG(L != nullptr && ms != nullptr, "layer or ms is NULL");
  CHECK_ARG(n_calls >= 0 && n_calls <= L->prof_n, "n_calls exceeds the timed calls kept");
  for (int c = 0; c < n_calls; ++c) {
    const cudaEvent_t* ev = &L->prof_ev[(size_t)c * (STARKV_N_PHASES + 1)];
    for (int p = 0; p < STARKV_N_PHASES; ++p) {
      float t = 0.f;
      if (L->prof_used[c]) {
        CUDA_TRY(cudaEventSynchronize(ev[p + 1]));
        CUDA_TRY(cudaEventElapsedTime(&t, ev[p], ev[p + 1]));
      }
      ms[(size_t)c * STARKV_N_PHASES + p] = t;
    }
  }
  return STARKV_OK;
}

starkv_status starkv_check_wait_timeout(const starkv_layer* L, uint32_t limit_us, starkv_stream_t stream) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  CHECK_ARG(limit_us >= 1 && limit_us <= 2000000, "limit_us must be in [1, 2000000]");
  CUDA_TRY(launch_wait_timeout_check(L->status, 1000ull * limit_us, (cudaStream_t)stream));
  return STARKV_OK;
}

starkv_status starkv_sync_status(const starkv_layer* L, starkv_stream_t stream, uint32_t* bits) {
  set_error("");
  CHECK_ARG(L != nullptr, "layer is NULL");
  uint32_t w = 0;
  cudaStream_t s = (cudaStream_t)stream;
  CUDA_TRY(cudaMemcpyAsync(&w, L->status, sizeof(w), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaMemsetAsync(L->status, 0, sizeof(uint32_t), s));
  CUDA_TRY(cudaStreamSynchronize(s));
  if (bits) *bits = w;
  if (w == 0) return STARKV_OK;
  if (w == STARKV_DEV_TIMEOUT) return STARKV_ERR_TIMEOUT;
  return STARKV_ERR_DEVICE;
}

}  // extern "C"
