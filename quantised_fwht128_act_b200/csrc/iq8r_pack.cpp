// Host-side round-to-nearest packing of bf16 weights into the IQ8R formats.
//
// Trunk ("Qwen3.8-27B IQ8R + DFlash2 -- radiance container", table row
// "Weights", and the recipe rule "codes=i8 group=256 scale=u8 scale2=bf16
// block2=1x* transform=fwht128 clamp=sym"): int8 codes -127..127; each row
// has a bf16 scale and, below it, a u8 sub-scale for every 256 of K; every
// 128 of K goes through the unnormalised Hadamard transform first.
// lm_head (same row; recipe "codes=i8 group=128 scale=bf16 clamp=sym"): a
// bf16 scale per (row, 128 of K).
//
// The pages fit the codes by GPTQ against calibration Hessians; packing here
// is the recipes' "rtn" rule with these stated scale definitions (and, on
// request, rule=search over the scales below them, see pack_range):
//   trunk:   s2 = bf16 of R / (127 * 255) rounded up, R the row's absmax;
//            s1 = min(255, ceil(A / (127 * s2))), A the 256-block's absmax;
//            code = clamp(rint(w' / (s2 * s1)), -127, 127).
//   lm_head: s = bf16 of A / 127 rounded up (A over the 128-block);
//            code = clamp(rint(w' / s), -127, 127).
// Every step is one IEEE float32 operation (this file must be compiled
// without fast-math or FMA contraction), so the bytes are reproducible.

#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "iq8r_internal.h"

namespace iq8r {
namespace {

inline float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

inline uint32_t float_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

inline float bits_float(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Smallest bf16 >= v for finite v >= 0: keep the upper 16 bits and step one
// bf16 unit up if anything was cut off (the same rule covers subnormals).
inline uint16_t bf16_round_up_bits(float v) {
  uint32_t u = float_bits(v);
  uint32_t hi = u & 0xFFFF0000u;
  if (u & 0x0000FFFFu) hi += 0x00010000u;
  return static_cast<uint16_t>(hi >> 16);
}

// In-place fwht128 on 128 floats: stages h = 1, 2, 4, ..., 64 in that order,
// (a, b) -> (a + b, a - b).
inline void fwht128(float* v) {
  for (int h = 1; h < kRot; h <<= 1) {
    for (int i = 0; i < kRot; i += 2 * h) {
      for (int j = i; j < i + h; ++j) {
        const float a = v[j];
        const float b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

inline int8_t quantise(float w, float step) {
  if (!(step > 0.0f)) return 0;
  float q = std::nearbyint(w / step);  // round-half-even (default mode)
  q = std::min(127.0f, std::max(-127.0f, q));
  return static_cast<int8_t>(q);
}

// Squared reconstruction error of one group at step `d`: (w' - code * d)^2
// in double, added in index order.
inline double group_sse(const float* v, int64_t len, float d) {
  double sse = 0.0;
  for (int64_t i = 0; i < len; ++i) {
    const double e = static_cast<double>(v[i]) - static_cast<double>(quantise(v[i], d)) * static_cast<double>(d);
    sse += e * e;
  }
  return sse;
}

// Index of the codebook level nearest to w / s (s > 0): the quotient in
// float32, the distances in double, ties going to the larger level.
inline uint8_t cb4_index(float w, float s) {
  const double t = static_cast<double>(w / s);
  double best = 1e300;
  uint8_t bi = 8;
  for (int c = 15; c >= 0; --c) {  // from the top: a tie keeps the larger level
    const double d = std::fabs(t - static_cast<double>(kCb4Table[c]));
    if (d < best) {
      best = d;
      bi = static_cast<uint8_t>(c);
    }
  }
  return bi;
}

// Squared reconstruction error of one codebook group at scale `s`:
// (w' - level * s)^2 in double, added in index order.
inline double cb4_sse(const float* v, int64_t len, float s) {
  double sse = 0.0;
  for (int64_t i = 0; i < len; ++i) {
    const double e = static_cast<double>(v[i]) - static_cast<double>(kCb4Table[cb4_index(v[i], s)]) *
                                                     static_cast<double>(s);
    sse += e * e;
  }
  return sse;
}

// The recipes' rule=search (one scale per 128 columns chosen by a search for
// the least error: "Qwen3.8-Flash-Next, IQR-V4 -- radiance container", row
// "Trunk"): the RTN step and the kSearchWindow - 1 next smaller ones, least
// error wins, ties to the larger step.
constexpr int kSearchWindow = 16;

void pack_range(int fmt, bool rotate, int rule, const uint16_t* w, int64_t k, int64_t r0, int64_t r1,
                int8_t* codes, uint8_t* sub, uint16_t* scale) {
  std::vector<float> row(static_cast<size_t>(k));
  const int64_t g256 = k / kGroupTrunk;
  const int64_t g128 = k / kGroupHead;
  std::vector<float> amax(static_cast<size_t>(std::max<int64_t>(g128, 1)));
  for (int64_t r = r0; r < r1; ++r) {
    const uint16_t* src = w + r * k;
    for (int64_t i = 0; i < k; ++i) row[i] = bf16_to_float(src[i]);
    if (rotate)
      for (int64_t c = 0; c < k; c += kRot) fwht128(row.data() + c);
    int8_t* out = codes + r * k;
    if (fmt == 0) {
      float R = 0.0f;
      for (int64_t g = 0; g < g256; ++g) {
        float A = 0.0f;
        for (int64_t i = g * kGroupTrunk; i < (g + 1) * kGroupTrunk; ++i) A = std::max(A, std::fabs(row[i]));
        amax[g] = A;
        R = std::max(R, A);
      }
      const uint16_t s2b = bf16_round_up_bits(R / 32385.0f);
      const float s2 = bf16_to_float(s2b);
      scale[r] = s2b;
      const float den = 127.0f * s2;  // exact: 7-bit x 8-bit significands
      for (int64_t g = 0; g < g256; ++g) {
        float s1 = 0.0f;
        if (s2 > 0.0f) s1 = std::min(255.0f, std::ceil(amax[g] / den));
        if (rule == 1 && s2 > 0.0f && s1 >= 1.0f) {
          const float* v = row.data() + g * kGroupTrunk;
          double best = group_sse(v, kGroupTrunk, s2 * s1);
          float best_s1 = s1;
          for (int i = 1; i < kSearchWindow && s1 - static_cast<float>(i) >= 1.0f; ++i) {
            const float c = s1 - static_cast<float>(i);
            const double e = group_sse(v, kGroupTrunk, s2 * c);
            if (e < best) {
              best = e;
              best_s1 = c;
            }
          }
          s1 = best_s1;
        }
        sub[r * g256 + g] = static_cast<uint8_t>(s1);
        const float d = s2 * s1;  // exact: 8-bit x 8-bit significands
        for (int64_t i = g * kGroupTrunk; i < (g + 1) * kGroupTrunk; ++i) out[i] = quantise(row[i], d);
      }
    } else if (fmt == 2) {
      // the drafter's codebook: nearest of 16 levels, two indices a byte
      uint8_t* pk = reinterpret_cast<uint8_t*>(codes) + r * (k / 2);
      for (int64_t g = 0; g < g128; ++g) {
        float A = 0.0f;
        for (int64_t i = g * kGroupHead; i < (g + 1) * kGroupHead; ++i) A = std::max(A, std::fabs(row[i]));
        uint16_t sb = bf16_round_up_bits(A / 127.0f);
        if (rule == 1 && sb > 0) {
          const float* v = row.data() + g * kGroupHead;
          double best = cb4_sse(v, kGroupHead, bf16_to_float(sb));
          uint16_t best_b = sb;
          for (int i = 1; i < kSearchWindow && static_cast<int>(sb) - i >= 1; ++i) {
            const uint16_t c = static_cast<uint16_t>(sb - i);  // the next smaller positive bf16
            const double e = cb4_sse(v, kGroupHead, bf16_to_float(c));
            if (e < best) {
              best = e;
              best_b = c;
            }
          }
          sb = best_b;
        }
        scale[r * g128 + g] = sb;
        const float s = bf16_to_float(sb);
        for (int64_t i = g * kGroupHead; i < (g + 1) * kGroupHead; i += 2) {
          const uint8_t lo = s > 0.0f ? cb4_index(row[i], s) : 8;
          const uint8_t hi = s > 0.0f ? cb4_index(row[i + 1], s) : 8;
          pk[i / 2] = static_cast<uint8_t>(lo | (hi << 4));
        }
      }
    } else {
      for (int64_t g = 0; g < g128; ++g) {
        float A = 0.0f;
        for (int64_t i = g * kGroupHead; i < (g + 1) * kGroupHead; ++i) A = std::max(A, std::fabs(row[i]));
        uint16_t sb = bf16_round_up_bits(A / 127.0f);
        if (rule == 1 && sb > 0) {
          const float* v = row.data() + g * kGroupHead;
          double best = group_sse(v, kGroupHead, bf16_to_float(sb));
          uint16_t best_b = sb;
          for (int i = 1; i < kSearchWindow && static_cast<int>(sb) - i >= 1; ++i) {
            const uint16_t c = static_cast<uint16_t>(sb - i);  // the next smaller positive bf16
            const double e = group_sse(v, kGroupHead, bf16_to_float(c));
            if (e < best) {
              best = e;
              best_b = c;
            }
          }
          sb = best_b;
        }
        scale[r * g128 + g] = sb;
        const float s = bf16_to_float(sb);
        for (int64_t i = g * kGroupHead; i < (g + 1) * kGroupHead; ++i) out[i] = quantise(row[i], s);
      }
    }
  }
}

}  // namespace

void pack_rows(int fmt, bool rotate, int rule, const uint16_t* w, int64_t n, int64_t k, int8_t* codes,
               uint8_t* sub, uint16_t* scale, int n_threads) {
  if (n_threads <= 0) n_threads = static_cast<int>(std::max(1u, std::thread::hardware_concurrency()));
  const int64_t per = std::max<int64_t>(64, (n + n_threads - 1) / n_threads);
  std::vector<std::thread> pool;
  for (int64_t r0 = 0; r0 < n; r0 += per) {
    const int64_t r1 = std::min(n, r0 + per);
    pool.emplace_back(pack_range, fmt, rotate, rule, w, k, r0, r1, codes, sub, scale);
  }
  for (auto& t : pool) t.join();
}

}  // namespace iq8r
