// Host-side check of the packed weight layout (compiled and run by
// tests/test_layout.py, no GPU needed): for every format, the map from
// element (n, k) to (byte, bit) is a bijection onto the packed bits, and the
// fields a lane reads for fragment register i of tensor-core step s are the
// elements that register must hold (rows g / g+8, K pairs in the order the
// activations are loaded).
#include <cstdio>
#include <vector>

#include "../mixed_gemm_b200/csrc/wq_internal.cuh"

using namespace wq;

static bool bijection(int f, int64_t N, int64_t K) {
  const int bits = code_bits(f);
  std::vector<int> used((size_t)(N * K * bits), 0);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t off;
      int sh;
      packed_loc(f, n, k, K, &off, &sh);
      for (int b = 0; b < bits; ++b) {
        const int64_t bit = off * 8 + sh + b;
        if (bit < 0 || bit >= (int64_t)used.size()) return false;
        used[(size_t)bit]++;
      }
    }
  for (int u : used)
    if (u != 1) return false;
  return true;
}

// 4-bit "magic" order and INT2: register i of step s of chunk c for lane
// (g, tq) holds rows g + 8*(i & 1), K = 32c + 8tq + 4s + 2*(i >> 1) + {0, 1}
// in the low / high 16 bits, at the bit the decoders shift by.
static bool fragments(int f) {
  const int64_t K = 64;
  for (int g = 0; g < 8; ++g)
    for (int tq = 0; tq < 4; ++tq)
      for (int c = 0; c < 2; ++c)
        for (int s = 0; s < 2; ++s)
          for (int i = 0; i < 4; ++i)
            for (int half = 0; half < 2; ++half) {
              const int64_t n = g + 8 * (i & 1), k = 32 * c + 8 * tq + 4 * s + 2 * (i >> 1) + half;
              int64_t off;
              int sh;
              packed_loc(f, n, k, K, &off, &sh);
              const int lane = 4 * g + tq;
              int64_t word_off;
              int want;
              if (f == INT2_SYM) {
                word_off = (int64_t)lane * 8 + c * 4;
                want = 2 * (4 * s + i) + 16 * half;
              } else {
                word_off = (int64_t)lane * 16 + (2 * c + s) * 4;
                want = 4 * i + 16 * half;
              }
              const int bit = (int)((off - word_off) * 8 + sh);
              if (off < word_off || off >= word_off + 4 || bit != want) return false;
            }
  return true;
}

// INT3: the low-plane field and the high-plane bit of every element cover
// each packed bit once, and the fields of fragment register i of step s of
// chunk c sit where frag_int3 reads them: low bits at 2 (4s + i) (+16) of the
// lane's word c, high bit at 8c + 4s + i (+16) of the lane's high word.
static bool int3_layout(int64_t N, int64_t K) {
  std::vector<int> used((size_t)(N * K * 3), 0);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t lo, hi;
      int ls, hs;
      packed_loc3(n, k, K, &lo, &ls, &hi, &hs);
      for (int b = 0; b < 2; ++b) {
        const int64_t bit = lo * 8 + ls + b;
        if (bit < 0 || bit >= (int64_t)used.size()) return false;
        used[(size_t)bit]++;
      }
      const int64_t hb = hi * 8 + hs;
      if (hb < 0 || hb >= (int64_t)used.size()) return false;
      used[(size_t)hb]++;
    }
  for (int u : used)
    if (u != 1) return false;
  for (int g = 0; g < 8; ++g)
    for (int tq = 0; tq < 4; ++tq)
      for (int c = 0; c < 2; ++c)
        for (int s = 0; s < 2; ++s)
          for (int i = 0; i < 4; ++i)
            for (int half = 0; half < 2; ++half) {
              const int64_t n = g + 8 * (i & 1), k = 32 * c + 8 * tq + 4 * s + 2 * (i >> 1) + half;
              int64_t lo, hi;
              int ls, hs;
              packed_loc3(n, k, 64, &lo, &ls, &hi, &hs);
              const int lane = 4 * g + tq;
              const int64_t lw = (int64_t)lane * 8 + c * 4, hw = 256 + (int64_t)lane * 4;
              if (lo < lw || lo >= lw + 4 || (lo - lw) * 8 + ls != 2 * (4 * s + i) + 16 * half)
                return false;
              if (hi < hw || hi >= hw + 4 || (hi - hw) * 8 + hs != 8 * c + 4 * s + i + 16 * half)
                return false;
            }
  return true;
}

int main() {
  int bad = 0;
  const int fmts[] = {INT4_SYM, INT4_ASYM, INT8_SYM, CB4, NVFP4, MXFP4, FP8_E4M3, FP8_E5M2,
                      INT2_SYM};
  for (int f : fmts) {
    const bool ok = bijection(f, 48, 192) && bijection(f, 16, 64);
    printf("format %d bijection %s\n", f, ok ? "ok" : "FAIL");
    bad += !ok;
  }
  {
    const bool ok = int3_layout(48, 192) && int3_layout(16, 64);
    printf("format %d two-plane layout and fragments %s\n", (int)INT3_SYM, ok ? "ok" : "FAIL");
    bad += !ok;
  }
  for (int f : {INT4_SYM, INT4_ASYM, NVFP4, MXFP4, INT2_SYM}) {
    const bool ok = fragments(f);
    printf("format %d fragments %s\n", f, ok ? "ok" : "FAIL");
    bad += !ok;
  }
  return bad;
}
