// Device copy of the seeded normal generator of synth/workloads.py.
//
// Same definition, same operation order: SplitMix64 outputs h(c) =
// mix64(key + (c + 1) * GAMMA); Box-Muller on pairs (u1 in (0,1], u2 in
// [0,1)); ln, cos and sin from the series in synth/workloads.py with the
// coefficient tables passed in from Python.  Compiled with -fmad=false so
// every + and * rounds separately, exactly as numpy evaluates them; the
// outputs are therefore bit-identical to the host generator.  Test-support
// code: it holds none of the attention arithmetic.

#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr int NTERMS = 12;

struct Series {
  double log_c[NTERMS];
  double cos_c[NTERMS];
  double sin_c[NTERMS];
  double ln2, half_pi, sqrt_half;
};

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ double log_series(double x, const Series& s) {
  int e;
  double m = frexp(x, &e);
  if (m < s.sqrt_half) {
    m = m * 2.0;
    e -= 1;
  }
  const double t = (m - 1.0) / (m + 1.0);
  const double t2 = t * t;
  double p = s.log_c[NTERMS - 1];
  for (int k = NTERMS - 2; k >= 0; --k) p = p * t2 + s.log_c[k];
  return static_cast<double>(e) * s.ln2 + (2.0 * t) * p;
}

__device__ void sincos_turn(double u, const Series& s, double* cos_t, double* sin_t) {
  const double w = u * 4.0;
  const double q = floor(w);
  const double a = (w - q) * s.half_pi;
  const double a2 = a * a;
  double c = s.cos_c[NTERMS - 1];
  for (int k = NTERMS - 2; k >= 0; --k) c = c * a2 + s.cos_c[k];
  double sn = s.sin_c[NTERMS - 1];
  for (int k = NTERMS - 2; k >= 0; --k) sn = sn * a2 + s.sin_c[k];
  sn = sn * a;
  const int qi = static_cast<int>(q) & 3;
  if (qi == 0) { *cos_t = c; *sin_t = sn; }
  else if (qi == 1) { *cos_t = -sn; *sin_t = c; }
  else if (qi == 2) { *cos_t = -c; *sin_t = -sn; }
  else { *cos_t = sn; *sin_t = -c; }
}

__device__ __forceinline__ uint16_t bf16_rne_bits(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  const uint16_t sign = static_cast<uint16_t>(b >> 63);
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
  const uint64_t r = mag + ((1ull << 44) - 1) + ((mag >> 45) & 1ull);
  const int64_t e32 = static_cast<int64_t>((r >> 52) & 0x7FF) - 1023 + 127;
  uint16_t frac = static_cast<uint16_t>((r >> 45) & 0x7F);
  uint16_t e16 = static_cast<uint16_t>(e32);
  if (e32 <= 0) { e16 = 0; frac = 0; }
  return static_cast<uint16_t>((sign << 15) | (e16 << 7) | frac);
}

// kind: 0 = float64, 1 = float32, 2 = bfloat16 bits
__global__ void normal_kernel(void* dst, long long start, long long count, unsigned long long key, int kind,
                              Series s) {
  const long long p0 = start / 2;
  const long long pair = p0 + static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (2 * pair >= start + count) return;
  const uint64_t h1 = mix64(key + static_cast<uint64_t>(2 * pair + 1) * 0x9E3779B97F4A7C15ull);
  const uint64_t h2 = mix64(key + static_cast<uint64_t>(2 * pair + 2) * 0x9E3779B97F4A7C15ull);
  const double u1 = static_cast<double>((h1 >> 11) + 1) * 0x1p-53;
  const double u2 = static_cast<double>(h2 >> 11) * 0x1p-53;
  const double r = sqrt(-2.0 * log_series(u1, s));
  double ct, st;
  sincos_turn(u2, s, &ct, &st);
  const double v[2] = {r * ct, r * st};
  for (int j = 0; j < 2; ++j) {
    const long long e = 2 * pair + j;
    if (e < start || e >= start + count) continue;
    const long long o = e - start;
    if (kind == 0) static_cast<double*>(dst)[o] = v[j];
    else if (kind == 1) static_cast<float*>(dst)[o] = __double2float_rn(v[j]);
    else static_cast<uint16_t*>(dst)[o] = bf16_rne_bits(v[j]);
  }
}

}  // namespace

extern "C" int synth_normal(void* dst, long long start, long long count, unsigned long long key, int kind,
                            const double* log_c, const double* cos_c, const double* sin_c, double ln2,
                            double half_pi, double sqrt_half, void* stream) {
  if (!dst || count < 0 || start < 0 || kind < 0 || kind > 2) return -1;
  if (count == 0) return 0;
  Series s;
  for (int i = 0; i < NTERMS; ++i) {
    s.log_c[i] = log_c[i];
    s.cos_c[i] = cos_c[i];
    s.sin_c[i] = sin_c[i];
  }
  s.ln2 = ln2;
  s.half_pi = half_pi;
  s.sqrt_half = sqrt_half;
  const long long pairs = (start + count + 1) / 2 - start / 2;
  const int threads = 256;
  const long long blocks = (pairs + threads - 1) / threads;
  if (blocks > 0x7FFFFFFFLL) return -1;
  normal_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      dst, start, count, key, kind, s);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
