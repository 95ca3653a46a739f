// CPU oracle in plain C++: one MoE FFN layer over NVFP4 experts, in fp64.
//
// TEST INFRASTRUCTURE ONLY.  The product library never links or calls it;
// only the tests, the package's smoke check and the bench's CPU-baseline leg
// load it (through oracle/cpp.py).  It shares no code with the GPU path.
//
// What it computes is the plain definition of a top-k MoE FFN layer as the
// FreeToken pages describe its pieces ("FreeToken model guide", MoE expert
// scheduling and --quant-backend moe.nvfp4; "sm89-moe-offload" fork README,
// "Production configuration"): the pages never write the layer down, so each
// step below is the plainest reading, the same one the numpy oracle
// (oracle/moe_layer.py, oracle/nvfp4.py) takes:
//
//   route    top-k of the fp32 logits (descending; equal logits -> lower id),
//            weights w_j = exp(l_j - m) / sum_S exp(l_i - m), m = max over S,
//            in fp64
//   permute  stable counting sort of pairs p = t*k + j by expert id
//   decode   W[n,k] = e2m1(code) * e4m3(scale[n][k/16]) * global, exact in fp64
//   expert   G = Wg x, U = Wu x, h = G * U / (1 + exp(-G)), o = Wd h  (fp64)
//   combine  y[t] = sum_j w_j * o_{t,j}  (fp64)
//   pack     fp32 weights -> NVFP4 with IEEE fp32 round-to-nearest steps
//   mxfp4    the MXFP4 expert format the pages list beside NVFP4 ("FlashML-org /
//            FreeToken" about page, quantization formats; model guide, CPU
//            executor formats): E2M1 elements sharing one E8M0 scale per 32,
//            as the OCP Microscaling Formats (MX) v1.0 specification defines
//            the format and its conversion from fp32
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fopenmp -shared -fPIC
// (oracle/build.py); -ffp-contract=off keeps every fp32 step of pack a
// separately rounded operation.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ------------------------------------------------------------- decode ---

// E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; exponent 0
// is subnormal (0 or 0.5).
double e2m1_value(int code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// E4M3, FN variant: bias 7, exponent 0 subnormal (m/8 * 2^-6), S.1111.111
// is NaN, no infinities (max 448).
double e4m3_value(int byte) {
  const int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
  if (e == 15 && m == 7) return std::nan("");
  const double mag = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// E8M0 (MX shared scale): 2^(byte - 127); 255 is NaN; no sign, no zero.
double e8m0_value(int byte) {
  return byte == 255 ? std::nan("") : std::ldexp(1.0, byte - 127);
}

struct Tables {
  double e2m1[16];
  double e4m3[256];
  Tables() {
    for (int c = 0; c < 16; ++c) e2m1[c] = e2m1_value(c);
    for (int b = 0; b < 256; ++b) e4m3[b] = e4m3_value(b);
  }
};
const Tables& tables() {
  static const Tables t;
  return t;
}

// One expert tensor [N, K] as stored in a slot: codes [N, K/2] (even k in
// the low nibble), scales [N, ld] bytes, one fp32 global scale.
//   NVFP4 (mx = false): e2m1(code) * e4m3(scale[k/16]) * global
//   MXFP4 (mx = true):  e2m1(code) * e8m0(scale[k/16]); the slot stores each
//                       32-block's E8M0 byte at both of its 16-K positions,
//                       and the MX value has no global factor
struct Tensor {
  const uint8_t* codes;
  const uint8_t* scales;
  double global;
  int N, K, ld;
  bool mx;
  double scale(int n, int k) const {
    const uint8_t b = scales[size_t(n) * ld + k / 16];
    return mx ? e8m0_value(b) : tables().e4m3[b] * global;
  }
  double at(int n, int k) const {
    const uint8_t byte = codes[size_t(n) * (K / 2) + k / 2];
    const int code = (k & 1) ? (byte >> 4) : (byte & 15);
    return tables().e2m1[code] * scale(n, k);
  }
  bool has_nan_scale() const {
    for (int n = 0; n < N; ++n)
      for (int b = 0; b < K / 16; ++b)
        if (std::isnan(scale(n, 16 * b))) return true;
    return false;
  }
};

// --------------------------------------------------------------- pack ---

// Index of the grid value nearest to v >= 0 (ties to the even index,
// saturating above the top).
int round_to_grid(double v, const double* grid, int n) {
  if (v >= grid[n - 1]) return n - 1;
  if (v <= grid[0]) return 0;
  int hi = 1;
  while (grid[hi] < v) ++hi;   // grid[hi-1] < v <= grid[hi]
  const double dlo = v - grid[hi - 1], dhi = grid[hi] - v;
  if (dhi < dlo) return hi;
  if (dlo < dhi) return hi - 1;
  return (hi % 2 == 0) ? hi : hi - 1;
}

// ------------------------------------------------------------- route ---

void route_token(const float* l, int E, int k, int32_t* ids, double* w) {
  std::vector<int> order(E);
  for (int e = 0; e < E; ++e) order[e] = e;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return l[a] > l[b]; });   // equal -> lower id
  const double m = double(l[order[0]]);
  double sum = 0.0;
  for (int j = 0; j < k; ++j) sum += std::exp(double(l[order[j]]) - m);
  for (int j = 0; j < k; ++j) {
    ids[j] = order[j];
    w[j] = std::exp(double(l[order[j]]) - m) / sum;
  }
}

}  // namespace

extern "C" {

// Value of an E2M1 code / an E4M3 byte (NaN for the NaN pattern).
double orc_e2m1_value(int code) { return tables().e2m1[code & 15]; }
double orc_e4m3_value(int byte) { return tables().e4m3[byte & 255]; }

// fp32 [N, K] -> codes [N, K/2], scales [N, ld] (padding zero), global.
//   g   = amax / 2688             (amax over the tensor; g = 1 if amax = 0)
//   r_b = amax_b / (6 g)          (amax_b over a 16-block)
//   s_b = E4M3 nearest-even, saturating
//   q   = E2M1(w / (dec(s_b) g)) nearest-even, saturating; sign follows w;
//         a block whose scale decodes to 0 stores code 0.
// Returns 0, or -1 if K is not a multiple of 16 or ld < K/16.
int orc_pack(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld, float* global) {
  if (K % 16 || ld < K / 16) return -1;
  const Tables& T = tables();
  double e4m3_pos[127], e2m1_pos[8];
  for (int i = 0; i < 127; ++i) e4m3_pos[i] = T.e4m3[i];
  for (int i = 0; i < 8; ++i) e2m1_pos[i] = T.e2m1[i];
  float amax = 0.0f;
  for (size_t i = 0; i < size_t(N) * K; ++i) amax = std::max(amax, std::fabs(w[i]));
  const float g = amax == 0.0f ? 1.0f : amax / 2688.0f;
  *global = g;
  const float six_g = 6.0f * g;
  for (int n = 0; n < N; ++n) {
    std::memset(scales + size_t(n) * ld, 0, ld);
    for (int b = 0; b < K / 16; ++b) {
      const float* blk = w + size_t(n) * K + 16 * b;
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i) amax_b = std::max(amax_b, std::fabs(blk[i]));
      const float r = amax_b / six_g;
      const int sc = round_to_grid(double(r), e4m3_pos, 127);
      scales[size_t(n) * ld + b] = uint8_t(sc);
      const float sval = float(T.e4m3[sc]);
      const float qden = sval * g;
      for (int i = 0; i < 16; i += 2) {
        int c[2];
        for (int h = 0; h < 2; ++h) {
          const float x = blk[i + h];
          if (sval == 0.0f) { c[h] = 0; continue; }
          const float v = x / qden;
          const int mag = round_to_grid(double(std::fabs(v)), e2m1_pos, 8);
          c[h] = mag | (std::signbit(v) ? 8 : 0);
        }
        codes[size_t(n) * (K / 2) + (16 * b + i) / 2] = uint8_t(c[0] | (c[1] << 4));
      }
    }
  }
  return 0;
}

// Value of an E8M0 byte (NaN for 255).
double orc_e8m0_value(int byte) { return e8m0_value(byte & 255); }

// fp32 [N, K] -> MXFP4: codes [N, K/2] (even k in the low nibble), E8M0
// scales [N, ld] (padding zero), one scale per 32-element block.  Per block
// (the MX conversion of a vector):
//   x_b = floor(log2(amax_b)) - 2     (2: the largest exponent of E2M1, whose
//                                      largest value is 1.5 * 2^2 = 6),
//         clamped to [-127, 127]; x_b = -127 when amax_b = 0
//   scale byte = x_b + 127
//   q   = E2M1(w / 2^x_b) nearest-even, saturating at 6; sign follows w.
// Returns 0; -1 if K is not a multiple of 32 or ld < K/32; -2 on a
// non-finite input.
int orc_pack_mxfp4(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld) {
  if (K % 32 || ld < K / 32) return -1;
  for (size_t i = 0; i < size_t(N) * K; ++i)
    if (!std::isfinite(w[i])) return -2;
  double e2m1_pos[8];
  for (int i = 0; i < 8; ++i) e2m1_pos[i] = tables().e2m1[i];
  for (int n = 0; n < N; ++n) {
    std::memset(scales + size_t(n) * ld, 0, ld);
    for (int b = 0; b < K / 32; ++b) {
      const float* blk = w + size_t(n) * K + 32 * b;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, double(std::fabs(blk[i])));
      int x = -127;
      if (amax > 0.0) {
        int e;
        std::frexp(amax, &e);        // amax = f * 2^e, f in [0.5, 1): floor(log2 amax) = e - 1
        x = std::min(127, std::max(-127, (e - 1) - 2));
      }
      scales[size_t(n) * ld + b] = uint8_t(x + 127);
      for (int i = 0; i < 32; i += 2) {
        int c[2];
        for (int h = 0; h < 2; ++h) {
          const double v = std::ldexp(double(blk[i + h]), -x);   // exact: a power-of-two scaling in fp64
          c[h] = round_to_grid(std::fabs(v), e2m1_pos, 8) | (std::signbit(v) ? 8 : 0);
        }
        codes[size_t(n) * (K / 2) + (32 * b + i) / 2] = uint8_t(c[0] | (c[1] << 4));
      }
    }
  }
  return 0;
}

// MXFP4 [N, K] -> fp64 values (exact): e2m1(code) * 2^(scale - 127).
// Returns 0, or -1 for bad sizes or a NaN scale byte.
int orc_decode_mxfp4(const uint8_t* codes, const uint8_t* scales, int N, int K, int ld, double* out) {
  if (K % 32 || ld < K / 32) return -1;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const uint8_t sb = scales[size_t(n) * ld + k / 32];
      if (sb == 255) return -1;
      const uint8_t byte = codes[size_t(n) * (K / 2) + k / 2];
      const int code = (k & 1) ? (byte >> 4) : (byte & 15);
      out[size_t(n) * K + k] = tables().e2m1[code] * e8m0_value(sb);
    }
  return 0;
}

// logits fp32 [T, E] -> ids int32 [T, k], weights fp64 [T, k].
int orc_route(const float* logits, int T, int E, int k, int32_t* ids, double* w) {
  if (k < 1 || k > E) return -1;
  for (int t = 0; t < T; ++t) route_token(logits + size_t(t) * E, E, k, ids + size_t(t) * k, w + size_t(t) * k);
  return 0;
}

// ids [T*k] -> offsets [E+1], perm_src [T*k] (row -> pair), pair_to_row.
int orc_permute(const int32_t* ids, int T, int k, int E, int32_t* offsets, int32_t* perm_src, int32_t* pair_to_row) {
  const int P = T * k;
  std::vector<int> count(E, 0);
  for (int p = 0; p < P; ++p) {
    if (ids[p] < 0 || ids[p] >= E) return -1;
    ++count[ids[p]];
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + count[e];
  std::vector<int> next(offsets, offsets + E);
  for (int p = 0; p < P; ++p) {   // ascending p: stable
    const int r = next[ids[p]]++;
    perm_src[r] = p;
    pair_to_row[p] = r;
  }
  return 0;
}

// The layer for the listed tokens: y [ntok, H] fp64.
//   x_bits   bf16 bit patterns [T, H]; logits fp32 [T, E]
//   experts  read from a host copy of the slot pool: expert e's tensor m
//            (0 gate [I, H], 1 up [I, H], 2 down [H, I]) has its codes at
//            pool + slot_table[e] * slot_bytes + codes_off[m], its scales at
//            ... + scales_off[m] (ld_scale[m] bytes per row) and its fp32
//            global scale at ... + global_off[m]
//   fmt      0: NVFP4 experts; 1: MXFP4 experts (see Tensor)
// Returns 0, -1 on a bad argument, -2 on a NaN scale byte, -3 on a
// non-resident (slot < 0) expert.
int orc_moe_layer(const uint16_t* x_bits, const float* logits, int T, int E, int k, int H, int I,
                  const int32_t* slot_table, const uint8_t* pool, int64_t slot_bytes, const int64_t* codes_off,
                  const int64_t* scales_off, const int64_t* global_off, const int32_t* ld_scale,
                  const int32_t* tokens, int ntok, int fmt, double* y) {
  if (k < 1 || k > E || H % 16 || I % 16 || (fmt != 0 && fmt != 1)) return -1;
  for (int i = 0; i < ntok; ++i)
    if (tokens[i] < 0 || tokens[i] >= T) return -1;
  int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < ntok; ++i) {
    const int t = tokens[i];
    std::vector<int32_t> ids(k);
    std::vector<double> w(k), x(H), gv(I), uv(I), hv(I), o(H);
    route_token(logits + size_t(t) * E, E, k, ids.data(), w.data());
    for (int c = 0; c < H; ++c) {
      uint32_t u = uint32_t(x_bits[size_t(t) * H + c]) << 16;
      float f;
      std::memcpy(&f, &u, 4);
      x[c] = double(f);
    }
    double* yt = y + size_t(i) * H;
    for (int c = 0; c < H; ++c) yt[c] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int slot = slot_table[ids[j]];
      if (slot < 0) {
#pragma omp atomic write
        status = -3;
        continue;
      }
      const uint8_t* base = pool + size_t(slot) * size_t(slot_bytes);
      Tensor W[3];
      const int rows[3] = {I, I, H}, cols[3] = {H, H, I};
      for (int m = 0; m < 3; ++m) {
        float gs;
        std::memcpy(&gs, base + global_off[m], 4);
        W[m] = Tensor{base + codes_off[m], base + scales_off[m], double(gs), rows[m], cols[m], ld_scale[m], fmt == 1};
        if (W[m].has_nan_scale()) {
#pragma omp atomic write
          status = -2;
        }
      }
      for (int n = 0; n < I; ++n) {
        double gs = 0.0, us = 0.0;
        for (int c = 0; c < H; ++c) {
          gs += W[0].at(n, c) * x[c];
          us += W[1].at(n, c) * x[c];
        }
        gv[n] = gs;
        uv[n] = us;
        hv[n] = gs * us / (1.0 + std::exp(-gs));
      }
      for (int r = 0; r < H; ++r) {
        double s = 0.0;
        for (int n = 0; n < I; ++n) s += W[2].at(r, n) * hv[n];
        o[r] = s;
      }
      for (int c = 0; c < H; ++c) yt[c] += w[j] * o[c];
    }
  }
  return status;
}

}  // extern "C"
