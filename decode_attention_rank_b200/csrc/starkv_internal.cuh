// Internal definitions shared by the host API and the kernels of libstarkv.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <string>
#include <vector>

#include "starkv.h"

namespace starkv {

// One quantization/rotation group of a latent (channels [start, start + n) at `bits`).
struct GroupDesc {
  int start;
  int n;
  int bits;      // 0 = unquantized latent (one group spanning the whole latent)
  int code_off;  // byte offset of this group's code block inside the latent block
};

// One stored latent of a token: key latent of a KV head, or the value latent.
struct LatentDesc {
  int width;        // r
  int block_off;    // byte offset of the latent block inside the page
  int n_groups;
  int group0;       // index of the first group in the group table
  int ch_off;       // offset of this latent in the concatenated latent vector
  int scale_bytes;  // bytes of the scale block (0 when unquantized)
  int cmajor;       // 1: channel-major (the value latent of a latent layer), see code_bit and elem_index
  int n_hi;         // quantized: channels of the first (high-precision) segment
  int gsize;        // quantized: channels per group (groups are cut from each segment's start)
};

constexpr int kPage = 16;

// First bit of the code of (slot, channel i) inside a group's code block of n
// channels at `bits` bits.  Key latents are slot-major: a token's codes of
// the group are one run.  The value latent is channel-major: the 16 codes of
// a channel are one field of 16 * bits bits, even slots first, odd slots
// after them (place (s % 2) * 8 + s / 2), so that one shift and mask of the
// field puts the codes of slots 2k and 2k + 1 side by side.
__host__ __device__ __forceinline__ uint32_t code_bit(int slot, int i, int n, int bits, int cmajor) {
  return cmajor ? (uint32_t)(i * kPage + (slot & 1) * (kPage / 2) + (slot >> 1)) * (uint32_t)bits
                : (uint32_t)(slot * n + i) * (uint32_t)bits;
}

// Element index of (slot, channel j) inside an unquantized latent block of
// `width` channels: slot-major [slot][j], or channel-major [j][slot] (the
// value latent of a latent layer, so that one channel's 16 tokens are
// contiguous for the value contraction).
__host__ __device__ __forceinline__ size_t elem_index(int slot, int j, int width, int cmajor) {
  return cmajor ? (size_t)j * kPage + slot : (size_t)slot * width + j;
}

// Device status bits (mirror of STARKV_DEV_* in the public header).
constexpr uint32_t kBadPage = STARKV_DEV_BAD_PAGE;
constexpr uint32_t kBadPos = STARKV_DEV_BAD_POSITION;
constexpr uint32_t kScaleOvf = STARKV_DEV_SCALE_OVF;
constexpr uint32_t kTimeout = STARKV_DEV_TIMEOUT;

constexpr float kLog2e = 1.4426950408889634f;

// Everything a kernel needs to read or write one layer's pages.
struct LayerView {
  int D, H, Hkv, d, group_q;  // group_q = H / Hkv
  int L;                      // latents per token
  int Ltot;                   // sum of widths
  int Rk;                     // sum of key widths
  int wv;                     // value width per query head: r_v (joint) or d (plain)
  int rv;                     // width of the value latent (plain: Hkv*d)
  int es;                     // element bytes of unquantized latents (4 or 2)
  int dtype;                  // STARKV_F32 / STARKV_BF16
  int quantized, plain, rope;
  int hadamard;
  float rope_log2_theta;      // log2(theta)
  float scale_log2;           // softmax scale * log2(e)
  long long page_bytes;
  const LatentDesc* lat;      // device tables
  const GroupDesc* grp;
  uint32_t* status;
};

// Stored value of channel j of latent `ld` for token slot `slot` of a page block.
__device__ __forceinline__ float latent_value(const LayerView& v, const uint8_t* blk, const LatentDesc& ld,
                                              int slot, int j) {
  if (!v.quantized) {
    const size_t o = elem_index(slot, j, ld.width, ld.cmajor);
    return v.es == 4 ? reinterpret_cast<const float*>(blk)[o]
                     : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(blk)[o]);
  }
  // groups of gsize channels from the start of each segment
  const int g = ld.gsize == 32 ? (j < ld.n_hi ? j >> 5 : ((ld.n_hi + 31) >> 5) + ((j - ld.n_hi) >> 5))
                               : (j < ld.n_hi ? j / ld.gsize : (ld.n_hi + ld.gsize - 1) / ld.gsize + (j - ld.n_hi) / ld.gsize);
  const GroupDesc gd = v.grp[ld.group0 + g];
  const float s = __half2float(reinterpret_cast<const __half*>(blk)[g * kPage + slot]);
  const uint32_t bit = code_bit(slot, j - gd.start, gd.n, gd.bits, ld.cmajor);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + gd.code_off) + (bit >> 5);
  const uint32_t sh = bit & 31;
  uint32_t u = w[0] >> sh;
  if (sh + gd.bits > 32) u |= w[1] << (32 - sh);
  u &= (1u << gd.bits) - 1u;
  return (float)((int)u - (1 << (gd.bits - 1))) * s;
}

// One MMA item of the tensor-core score kernel: consecutive query heads whose
// W'' rows (sum of ranks <= 128) form the B operand of one 128 x npad MMA.
struct ScoreItem {
  int h0, nh, npad;   // first query head, heads, MMA N (multiple of 16)
  int w_off;          // byte offset of the item's W'' block in one sequence's W'' buffer
  int key_off;        // byte range of the item's key latent blocks inside a page
  int key_bytes;
  int hcol[8];        // G column of each head's first latent channel
  int hr[8];          // rank of each head
};

// The score epilogue's view of one query head: where its G columns and its
// key latent block are, and which compiled channel shape reads them (the
// shape fixes the block's layout).
struct ScoreHead {
  int gcol;          // G column of the head's first latent channel (item-relative)
  int kind;          // index of the compiled (hi channels, lo channels) shape
  int blk_rel;       // byte offset of the key latent block, relative to the item's key range in a page
  int run;           // GQA: heads from this one on in the item that share its KV head (1 .. 4; 0 inside a run)
};

// Outputs of the tensor-core score kernel.
struct ScoreOut {
  __half* P;          // [B][H][P_ld] exp2(s - m) with m the maximum of the token's 32-token group, fp16
  float* m_st;        // [B][H][n_g] per 32-token group
  long long P_ld;
  int n_st;           // 256-token super-tiles per sequence
  int n_g;            // 32-token groups per sequence
};

}  // namespace starkv

struct starkv_layer {
  starkv_layer_config cfg;
  std::vector<int> key_ranks;
  std::vector<starkv::LatentDesc> lat;
  std::vector<starkv::GroupDesc> grp;
  std::vector<int> key_off;     // prefix sums of key widths, size Hkv + 1
  starkv::LayerView view;
  size_t page_bytes = 0;
  double bytes_per_token = 0;
  size_t factor_bytes = 0;
  int device = 0;
  // device allocations owned by the layer
  starkv::LatentDesc* d_lat = nullptr;
  starkv::GroupDesc* d_grp = nullptr;
  int* d_key_off = nullptr;
  int* d_grp_lat = nullptr;     // latent index of every group
  void* A_T = nullptr;          // [Ltot][D] dtype: projection rows (unrotated)
  void* A_tiles = nullptr;      // bf16 layers: A_T as fp16 128x64 swizzled tiles (tensor-core projection)
  float* Bk = nullptr;          // [Rk][d] fp32: rotated key up-projections B' = R^T B
  // Fused output factors.  f32 layers: [D][H * wv] float32, row-major.  bf16
  // layers: fp16 tiles [Dp/128][Kp/64] of 128 x 64 elements, 128-byte swizzled
  // (the A operand of the tensor-core output kernel), zero padded.
  void* M_T = nullptr;
  int Kp = 0, Dp = 0;           // H * wv and D rounded up to 64 and 128
  // unfused output (config unfused_output = 1): no M; y_h B'_v,kv(h) then W_o on the tensor cores
  int unfused = 0;
  void* Bv_tiles = nullptr;     // fp16 tiles [H][r_v / 64] of 128 x 64: row p, column j = B'_v[j][kv(h) d + p]
  void* Wo_tiles = nullptr;     // fp16 tiles [Dp / 128][H d / 64] of 128 x 64: row n, column k = W_o[k][n]
  void* Bk_tiles = nullptr;     // prefill: per KV head one fp16 128 x 64 tile, row p, column j = B'_k[j][p] (j < r <= 64)
  uint32_t* status = nullptr;
  // tensor-core score kernel
  bool tc_scores = false;
  std::vector<starkv::ScoreItem> items;
  starkv::ScoreItem* d_items = nullptr;
  std::vector<starkv::ScoreHead> score_heads;   // one per query head
  starkv::ScoreHead* d_score_heads = nullptr;
  long long w_stride = 0;
  int w_stage = 0, k_stage = 0, WS = 0, KS = 0;
  int rope_tiles = 0;
  void* rope_E = nullptr;       // RoPE table tiles, 32 KB per 128 positions
  int decode_path = 0;          // 0 auto, 1 CUDA cores, 2 tensor-core scores + CUDA-core values
  // tensor-core value kernel
  bool tc_values = false;
  int vblk_off = 0, vblk_bytes = 0;
  int val_raw = 0;              // raw page stages of the value kernel
  int val_na = 0;               // pages of A tiles the value kernel keeps in TMEM
  bool val_bf16 = false;        // the value latent is unquantized bf16 (channel-major)
  // optional per-kernel timing of the tensor-core decode: prof_n sets of
  // STARKV_N_PHASES + 1 events, the decode call number prof_calls picks the set
  std::vector<cudaEvent_t> prof_ev;
  int prof_n = 0;
  long long prof_calls = 0;
  std::vector<char> prof_used;
};

namespace starkv {

void set_error(const std::string& msg);

// Kernel launchers (defined in the .cu files).
cudaError_t launch_transpose_into(const void* src, int rows, int cols, int dtype, void* dst, int dst_row0,
                                  int dst_ld, cudaStream_t s);
cudaError_t launch_rotate_rows(const starkv_layer* L, const void* B, int dtype, int latent, int cols, float* out,
                               cudaStream_t s);
cudaError_t launch_fold_M(const starkv_layer* L, const float* Bv_rot, const void* W_o, cudaStream_t s);

cudaError_t launch_wait_timeout_check(uint32_t* status, unsigned long long limit_ns, cudaStream_t s);

cudaError_t launch_project(const starkv_layer* L, const void* x, int n, float* z, cudaStream_t s);
cudaError_t launch_pack(const starkv_layer* L, uint8_t* pool, long long n_pages, const int32_t* page_table,
                        int n_seqs, int max_pages, int n, const int32_t* seq_idx, const int32_t* positions, const float* z,
                        int rotate, int rope_keys, cudaStream_t s);

// Generic decode path: rows are (sequence, query position, visible length) triples.
struct RowInfo {
  const int32_t* row_seq;   // [rows] sequence of each row, or null = identity
  const int32_t* row_len;   // [rows] visible tokens (decode: seq_lens)
  const int32_t* row_pos;   // [rows] RoPE position of the query, or null = len - 1
};
cudaError_t launch_decode_generic(const starkv_layer* L, const uint8_t* pool, long long n_pages,
                                  const int32_t* page_table, int max_pages, int rows, RowInfo ri, int max_len,
                                  const void* q, void* out, void* ws, size_t ws_bytes, bool prefill,
                                  cudaStream_t s, bool tc_scores = false);
size_t decode_generic_ws_bytes(const starkv_layer* L, int rows, int max_len, bool prefill);

// Uncompressed bf16 layers with head_dim 128: a streaming CUDA-core decode
// writing split partials (pY [rows][n_splits][H][128], pm, pl) for the merge.
bool plain_decode_supported(const LayerView& v);
cudaError_t launch_plain_decode(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                                int max_pages, int rows, RowInfo ri, const float* qrot, int n_splits, int chunk,
                                float* pY, float* pm, float* pl, cudaStream_t s);

int num_sms();

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device.  The attribute is per (function, device); the last value set is
// remembered per pair so that repeated launches skip the call.
cudaError_t set_smem_limit(const void* kernel, size_t bytes);

bool plan_scores_tc(starkv_layer* L);
bool plan_values_tc(starkv_layer* L);
size_t values_tc_ws_bytes(const starkv_layer* L, int batch, int max_len);
cudaError_t launch_values_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const ScoreOut& so, void* ws,
                             void* ytiles, cudaStream_t s, cudaEvent_t ev_mid);
// `profile`: record the phase events of starkv_profile_decode (decode calls only).
cudaError_t launch_decode_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                             void* out, void* ws, size_t ws_bytes, cudaStream_t s, bool profile = true);
size_t decode_tc_ws_bytes(const starkv_layer* L, int batch, int max_len);
cudaError_t build_rope_table(starkv_layer* L, cudaStream_t s);
size_t scores_tc_ws_bytes(const starkv_layer* L, int batch, int max_len);
cudaError_t launch_scores_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                             void* ws, ScoreOut* out, float* S_dbg, long long S_ld, cudaStream_t s);

// Tensor-core output kernel (bf16 layers).
struct OutGeom {
  int KT, DT, G, slots;
};
int outproj_nb(int rows);
OutGeom gemm_geom(int n_out, int K);
size_t gemm_part_bytes(int n_out, int K, int rows);
size_t outproj_part_bytes(const starkv_layer* L, int rows);
// out[row][n] = sum_k y[row][k] Mt[n][k] with Mt as fp16 128x64 swizzled tiles, y as fp16 B tiles.
// y_group != 0: a block-diagonal (grouped) product, output tile dt (128 outputs) contracting only
// y's k-range [dt * K, dt * K + K) (y has n_out / 128 * K columns).
cudaError_t launch_gemm_tc(const uint8_t* Mt, int n_out, int K, int n_valid, const void* y_tiles, int rows,
                           void* out, bool out_f32, float* part, uint32_t* status, cudaStream_t s, int y_group = 0);
// Rows of a bf16 matrix as fp16 swizzled tiles of nb rows x 64 columns (nb = 0: the B-tile height for `rows`).
cudaError_t launch_pack_rows_tiles(const void* x, int rows, int K, void* tiles, cudaStream_t s, int nb = 0);
cudaError_t launch_pack_rows_tiles_f32(const float* x, int rows, int K, void* tiles, cudaStream_t s, int nb = 0);
// Tensor-core causal prefill (k_prefill.cu): one chunk of one sequence.
bool prefill_flash_supported(const starkv_layer* L);
cudaError_t launch_prefill_bk_tiles(const starkv_layer* L, void* tiles, cudaStream_t s);
size_t prefill_flash_ws_bytes(const starkv_layer* L, int max_T, int max_q);
cudaError_t launch_prefill_flash(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt_row,
                                 int q_start, int q_len, const void* q, void* out, void* ws, int max_T, int max_q,
                                 cudaStream_t s);
// Unfused output factors: B'_v,kv(h) per query head as 128 x 64 fp16 tiles [H][r_v / 64], and W_o^T
// as tiles [Dp / 128][H d / 64] (built from the same inputs as M).
cudaError_t launch_build_unfused(starkv_layer* L, const float* Bv_rot, const void* W_o, cudaStream_t s);
size_t rows_tiles_bytes(int rows, int K);
cudaError_t launch_outproj_tc(const starkv_layer* L, const void* y_tiles, int rows, void* out, float* part,
                              cudaStream_t s);

}  // namespace starkv
