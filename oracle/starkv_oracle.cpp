// Oracle for STAR-KV latent decode attention: a plain, slow float64 host C++
// implementation (TEST INFRASTRUCTURE).
//
// Only the tests, the package smoke check and the CPU baseline arm of the
// benchmark may load this library (through oracle/cpp.py).  The decode
// library never links it, and it shares no code with the CUDA path.  It is
// the same plain definition as the numpy oracle (oracle/starkv_oracle.py),
// written out independently, and the tests hold the two equal.
//
// What it computes (page titles and sections of the STAR-KV material):
//   * "STAR-KV 阅读笔记" section 2.2: latents Z = X A, factors A = U_r S_r,
//     B = V_r^T; sections 5.1-5.2: head-wise keys, joint values; section 5.3:
//     pre-RoPE key latents (each reconstructed key rotated by its own
//     position); section 6.1: block-wise Hadamard before quantization,
//     absorbed into the factors, high-magnitude block at 4 bits, the rest at
//     3 bits; Algorithm 2: the decode data flow.
//   * The model card "tenosra/longchat-7b-starkv-proxima": top_fraction 0.25,
//     4 and 3 bits.
// Readings where the pages are silent are the numpy oracle's (quantizer,
// segments and groups, rotation blocks, page format, RoPE pairing, GQA map).
//
// Attention is the plain definition over the reconstructed, dequantized K/V:
//     K_h = Zhat_k,kv(h) B'_k,kv(h),  V = Zhat_v B'_v,
//     out = sum_h softmax(RoPE(q_h) . RoPE(K_h)^T / sqrt(d)) V_kv(h) W_o,h
// with no fusion, no re-association and no split over tokens.  Heads are
// computed by separate threads (std::thread), each head in float64.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <thread>
#include <vector>

extern "C" {

struct OrcSpec {
  int hidden, n_heads, n_kv_heads, head_dim;
  int quantized;
  double top_fraction;
  int top_bits, bottom_bits, group_size;
  int hadamard;
  int rope;
  double rope_theta;
  int page_size;
};

// ---------------------------------------------------------------- segments and groups (section 6.1)
int orc_n_high(int r, double top_fraction) { return (int)ceil(top_fraction * r - 1e-9); }

// Groups of a latent of width r: (start, n, bits) triples into out (room for r triples); returns the count.
int orc_groups(int r, const OrcSpec* s, int* out) {
  if (!s->quantized) {
    out[0] = 0;
    out[1] = r;
    out[2] = 0;
    return 1;
  }
  const int nh = orc_n_high(r, s->top_fraction);
  const int seg_start[2] = {0, nh}, seg_len[2] = {nh, r - nh}, seg_bits[2] = {s->top_bits, s->bottom_bits};
  int k = 0;
  for (int seg = 0; seg < 2; ++seg)
    for (int x = 0; x < seg_len[seg]; x += s->group_size) {
      out[3 * k] = seg_start[seg] + x;
      out[3 * k + 1] = std::min(s->group_size, seg_len[seg] - x);
      out[3 * k + 2] = seg_bits[seg];
      ++k;
    }
  return k;
}

// ---------------------------------------------------------------- rotation (section 6.1)
// Unnormalised Sylvester-Hadamard entry (i, j) of order 2^k: (-1)^popcount(i & j).
static double sylvester_entry(int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0; }

// Direct sum of normalised Sylvester blocks over the binary decomposition of n (largest first), n x n.
void orc_group_rotation(int n, double* out) {
  memset(out, 0, sizeof(double) * (size_t)n * n);
  int k = 0;
  while (k < n) {
    int p = 1;
    while (p * 2 <= n - k) p *= 2;
    const double norm = 1.0 / sqrt((double)p);
    for (int i = 0; i < p; ++i)
      for (int j = 0; j < p; ++j) out[(size_t)(k + i) * n + (k + j)] = sylvester_entry(i, j) * norm;
    k += p;
  }
}

// Block-diagonal rotation of one latent (r x r): the group rotations on the diagonal; identity when off.
void orc_rotation(int r, const OrcSpec* s, double* out) {
  memset(out, 0, sizeof(double) * (size_t)r * r);
  if (!(s->quantized && s->hadamard)) {
    for (int i = 0; i < r; ++i) out[(size_t)i * r + i] = 1.0;
    return;
  }
  std::vector<int> g(3 * (size_t)r);
  const int ng = orc_groups(r, s, g.data());
  for (int x = 0; x < ng; ++x) {
    const int st = g[3 * x], n = g[3 * x + 1];
    std::vector<double> b((size_t)n * n);
    orc_group_rotation(n, b.data());
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) out[(size_t)(st + i) * r + st + j] = b[(size_t)i * n + j];
  }
}

// ---------------------------------------------------------------- number formats (IEEE-754 definitions)
static uint32_t f2u(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  return u;
}
static float u2f(uint32_t u) {
  float x;
  memcpy(&x, &u, 4);
  return x;
}

// float32 -> bfloat16 (round to nearest, ties to even), returned as float32.
float orc_bf16_round(float x) {
  const uint32_t u = f2u(x);
  const uint32_t lsb = (u >> 16) & 1u;
  return u2f((u + 0x7FFFu + lsb) & 0xFFFF0000u);
}

// Value of a binary16 bit pattern.
double orc_half_value(uint16_t h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  const double sgn = (h & 0x8000) ? -1.0 : 1.0;
  if (e == 0) return sgn * ldexp((double)m, -24);
  if (e == 31) return m ? NAN : sgn * INFINITY;
  return sgn * ldexp(1024.0 + m, e - 25);
}

// Smallest binary16 >= x (x finite, 0 <= x <= 65504): binary search over the ordered positive patterns.
uint16_t orc_fp16_round_up(float x) {
  uint16_t lo = 0, hi = 0x7BFF;   // +0 .. 65504
  if ((double)x <= 0.0) return 0;
  while (lo < hi) {
    const uint16_t mid = (uint16_t)((lo + hi) / 2);
    if (orc_half_value(mid) >= (double)x)
      hi = mid;
    else
      lo = (uint16_t)(mid + 1);
  }
  return lo;
}

// ---------------------------------------------------------------- quantizer (section 6.1 + readings)
// One (token, group) vector of float32 latents -> fp16 scale bits and offset-binary codes.
// Returns 1 (and writes nothing) when amax / qmax exceeds the largest fp16.
int orc_quantize_group(const float* z, int n, int bits, uint16_t* s16, uint8_t* u) {
  const int qmax = (1 << (bits - 1)) - 1;
  float amax = 0.f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, fabsf(z[i]));
  const float s32 = amax / (float)qmax;   // IEEE float32 division
  if (!(s32 <= 65504.f)) return 1;
  const uint16_t h = orc_fp16_round_up(s32);
  const float sf = (float)orc_half_value(h);
  for (int i = 0; i < n; ++i) {
    long q = 0;
    if (sf != 0.f) {
      q = lrintf(z[i] / sf);   // round half to even (default rounding mode), float32 division
      q = std::min<long>(std::max<long>(q, -qmax), qmax);
    }
    u[i] = (uint8_t)(q + (1 << (bits - 1)));
  }
  *s16 = h;
  return 0;
}

// ---------------------------------------------------------------- page format
static size_t ru(size_t x, size_t m) { return (x + m - 1) / m * m; }

size_t orc_block_bytes(int r, const OrcSpec* s, int elem_size) {
  const int P = s->page_size;
  if (!s->quantized) return ru((size_t)P * r * elem_size, 16);
  std::vector<int> g(3 * (size_t)r);
  const int ng = orc_groups(r, s, g.data());
  size_t total = ru((size_t)ng * P * 2, 16);
  for (int x = 0; x < ng; ++x) total += ru((size_t)P * g[3 * x + 1] * g[3 * x + 2] / 8, 16);
  return total;
}

// First stream bit of the code of (slot, channel i): key latents slot-major, the value latent
// channel-major with the even slots of a channel's field first.
static size_t code_bit(int slot, int i, int n, int bits, int P, int channel_major) {
  if (channel_major) return ((size_t)i * P + (size_t)(P / 2) * (slot % 2) + slot / 2) * bits;
  return ((size_t)slot * n + i) * bits;
}

// Bytes of one quantized latent block for Z [P][r] float32 (rows that hold NaN are empty slots).
// Returns 1 on a scale overflow.  Unquantized blocks are not produced here (they are plain element arrays).
int orc_pack_block(const float* Z, int r, const OrcSpec* s, int channel_major, uint8_t* out) {
  const int P = s->page_size;
  memset(out, 0, orc_block_bytes(r, s, 2));
  std::vector<int> g(3 * (size_t)r);
  const int ng = orc_groups(r, s, g.data());
  size_t code_off = ru((size_t)ng * P * 2, 16);
  std::vector<uint8_t> u(32);
  for (int x = 0; x < ng; ++x) {
    const int st = g[3 * x], n = g[3 * x + 1], bits = g[3 * x + 2];
    uint8_t* cb = out + code_off;
    for (int slot = 0; slot < P; ++slot) {
      const float* z = Z + (size_t)slot * r;
      bool empty = false;
      for (int i = 0; i < r; ++i)
        if (isnan(z[i])) empty = true;
      if (empty) continue;
      uint16_t h;
      u.resize(n);
      if (orc_quantize_group(z + st, n, bits, &h, u.data())) return 1;
      out[(x * P + slot) * 2] = (uint8_t)(h & 0xFF);
      out[(x * P + slot) * 2 + 1] = (uint8_t)(h >> 8);
      for (int i = 0; i < n; ++i) {
        const size_t b0 = code_bit(slot, i, n, bits, P, channel_major);
        for (int t = 0; t < bits; ++t)   // LSB first, one bit at a time
          if ((u[i] >> t) & 1u) cb[(b0 + t) / 8] |= (uint8_t)(1u << ((b0 + t) % 8));
      }
    }
    code_off += ru((size_t)P * n * bits / 8, 16);
  }
  return 0;
}

// Values a reader of the cache sees for float32 latents Z [T][r], float64: dequantized codes
// (u - 2^(b-1)) * scale, or the bf16 / float32 value when unquantized (elem_size 2 / 4).
int orc_stored_values(const float* Z, int T, int r, const OrcSpec* s, int elem_size, double* out) {
  if (!s->quantized) {
    for (size_t i = 0; i < (size_t)T * r; ++i) out[i] = elem_size == 2 ? (double)orc_bf16_round(Z[i]) : (double)Z[i];
    return 0;
  }
  std::vector<int> g(3 * (size_t)r);
  const int ng = orc_groups(r, s, g.data());
  std::vector<uint8_t> u(r);
  for (int t = 0; t < T; ++t)
    for (int x = 0; x < ng; ++x) {
      const int st = g[3 * x], n = g[3 * x + 1], bits = g[3 * x + 2];
      uint16_t h;
      if (orc_quantize_group(Z + (size_t)t * r + st, n, bits, &h, u.data())) return 1;
      const double sc = orc_half_value(h);
      for (int i = 0; i < n; ++i) out[(size_t)t * r + st + i] = ((double)u[i] - (double)(1 << (bits - 1))) * sc;
    }
  return 0;
}

// ---------------------------------------------------------------- RoPE (rotate-half pairing)
// Row x (d values) rotated by position pos: pairs (p, p + d/2), theta_p = theta^(-2p/d).
static void rope_row(const double* x, int d, double pos, double theta, double* y) {
  const int half = d / 2;
  for (int p = 0; p < half; ++p) {
    const double ang = pos * pow(theta, -2.0 * p / d);
    const double c = cos(ang), sn = sin(ang);
    const double a = x[p], b = x[p + half];
    y[p] = a * c - b * sn;
    y[p + half] = b * c + a * sn;
  }
}

void orc_rope(const double* x, int n, int d, const double* pos, double theta, double* out) {
  for (int i = 0; i < n; ++i) rope_row(x + (size_t)i * d, d, pos[i], theta, out + (size_t)i * d);
}

// ---------------------------------------------------------------- attention (Algorithm 2, plain definition)
// Zk[g]: stored key latents of KV head g [T][r_g]; Bk[g]: B'_k,g [r_g][d]; Zv [T][r_v]; Bv [r_v][H_kv d];
// Wo [H d][D]; q [H][d].  Keys 0 .. seq_len - 1 are attended to; the query is at q_pos.  out [D].
void orc_decode(const OrcSpec* s, const int* key_ranks, const double* const* Zk, const double* const* Bk,
                const double* Zv, int rv, const double* Bv, const double* Wo, const double* q, int q_pos, int seq_len,
                int n_threads, double* out) {
  const int H = s->n_heads, Hkv = s->n_kv_heads, d = s->head_dim, D = s->hidden, T = seq_len;
  const int gq = H / Hkv;
  const double scale = 1.0 / sqrt((double)d);
  std::vector<std::vector<double>> part(H, std::vector<double>(D, 0.0));
  auto head = [&](int h) {
    const int g = h / gq;   // GQA: contiguous groups of query heads per KV head
    const int r = key_ranks[g];
    // K_h = Zhat_k,g B'_k,g, explicit [T][d]; RoPE at slot positions
    std::vector<double> K((size_t)T * d, 0.0), Kr((size_t)T * d), qr(d);
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < r; ++j) {
        const double z = Zk[g][(size_t)t * r + j];
        for (int p = 0; p < d; ++p) K[(size_t)t * d + p] += z * Bk[g][(size_t)j * d + p];
      }
    if (s->rope) {
      for (int t = 0; t < T; ++t) rope_row(&K[(size_t)t * d], d, (double)t, s->rope_theta, &Kr[(size_t)t * d]);
      rope_row(q + (size_t)h * d, d, (double)q_pos, s->rope_theta, qr.data());
    } else {
      Kr = K;
      for (int p = 0; p < d; ++p) qr[p] = q[(size_t)h * d + p];
    }
    // max-subtracted softmax
    std::vector<double> sc(T);
    double m = -INFINITY;
    for (int t = 0; t < T; ++t) {
      double a = 0.0;
      for (int p = 0; p < d; ++p) a += qr[p] * Kr[(size_t)t * d + p];
      sc[t] = a * scale;
      m = std::max(m, sc[t]);
    }
    double den = 0.0;
    for (int t = 0; t < T; ++t) den += (sc[t] = exp(sc[t] - m));
    // V_g = Zhat_v B'_v[:, g d .. (g+1) d], explicit [T][d]; y = p V_g; out += y W_o,h
    std::vector<double> V((size_t)T * d, 0.0), y(d, 0.0);
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < rv; ++j) {
        const double z = Zv[(size_t)t * rv + j];
        const double* brow = Bv + (size_t)j * Hkv * d + (size_t)g * d;
        for (int p = 0; p < d; ++p) V[(size_t)t * d + p] += z * brow[p];
      }
    for (int t = 0; t < T; ++t)
      for (int p = 0; p < d; ++p) y[p] += (sc[t] / den) * V[(size_t)t * d + p];
    for (int p = 0; p < d; ++p)
      for (int n = 0; n < D; ++n) part[h][n] += y[p] * Wo[(size_t)(h * d + p) * D + n];
  };
  const int nt = std::max(1, std::min(n_threads, H));
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w)
    pool.emplace_back([&, w]() {
      for (int h = w; h < H; h += nt) head(h);
    });
  for (auto& th : pool) th.join();
  for (int n = 0; n < D; ++n) {
    double a = 0.0;
    for (int h = 0; h < H; ++h) a += part[h][n];   // fixed order over heads
    out[n] = a;
  }
}

// Uncompressed layer (the protected layers): stored K (already rotated by RoPE) and V, [T][H_kv d] each.
void orc_decode_plain(const OrcSpec* s, const double* Khat, const double* Vhat, const double* Wo, const double* q,
                      int q_pos, int seq_len, double* out) {
  const int H = s->n_heads, Hkv = s->n_kv_heads, d = s->head_dim, D = s->hidden, T = seq_len;
  const int gq = H / Hkv;
  std::vector<double> qr(d), sc(T), y(d);
  for (int n = 0; n < D; ++n) out[n] = 0.0;
  for (int h = 0; h < H; ++h) {
    const int g = h / gq;
    if (s->rope)
      rope_row(q + (size_t)h * d, d, (double)q_pos, s->rope_theta, qr.data());
    else
      for (int p = 0; p < d; ++p) qr[p] = q[(size_t)h * d + p];
    double m = -INFINITY;
    for (int t = 0; t < T; ++t) {
      double a = 0.0;
      for (int p = 0; p < d; ++p) a += qr[p] * Khat[(size_t)t * Hkv * d + (size_t)g * d + p];
      sc[t] = a / sqrt((double)d);
      m = std::max(m, sc[t]);
    }
    double den = 0.0;
    for (int t = 0; t < T; ++t) den += (sc[t] = exp(sc[t] - m));
    for (int p = 0; p < d; ++p) {
      double a = 0.0;
      for (int t = 0; t < T; ++t) a += (sc[t] / den) * Vhat[(size_t)t * Hkv * d + (size_t)g * d + p];
      y[p] = a;
    }
    for (int p = 0; p < d; ++p)
      for (int n = 0; n < D; ++n) out[n] += y[p] * Wo[(size_t)(h * d + p) * D + n];
  }
}

}  // extern "C"
