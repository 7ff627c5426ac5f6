// NF4 level table, built on the host from the quantile formula.
//
// "QLoRA: Quantize Base Weights to 4-Bit", §2.1: q_i = (Q(i/(2^k+1)) +
// Q((i+1)/(2^k+1))) / 2 with Q the standard-normal quantile, k = 4.
// "QLoRA — Fine-Tuning a 65B Model on One GPU", "NF4: sixteen levels shaped
// like the weights": 8 negative and 8 non-negative levels, an exact 0,
// endpoints -1 and +1.  The formula cannot give 16 finite levels as printed
// (Q(0) = -inf at i = 0), so it is applied to each half:
//   non-negative half: D = 17, i = 8..15 (i = 8 is 0 by symmetry), scaled so
//   the i = 15 level is 1;
//   negative half: D = 19, i = 10..17 (i = 9 would again be 0), mirrored and
//   scaled so the i = 17 level is -1.
// The quantile is computed by bisection on Phi(x) = erfc(-x/sqrt 2)/2 in double
// and polished by Newton steps; the level is then rounded to fp32.
#include <cmath>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace ql {
namespace {

double phi_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double phi_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    if (phi_cdf(mid) < p) lo = mid; else hi = mid;
  }
  double x = 0.5 * (lo + hi);
  const double inv_sqrt_2pi = 0.39894228040143267794;
  for (int i = 0; i < 3; ++i) {
    double dens = inv_sqrt_2pi * std::exp(-0.5 * x * x);
    x -= (phi_cdf(x) - p) / dens;
  }
  return x;
}

double level(double D, int i) { return 0.5 * (phi_quantile(i / D) + phi_quantile((i + 1) / D)); }

NF4Table build() {
  NF4Table t{};
  const double top = level(17.0, 15);
  const double bottom = level(19.0, 17);
  for (int i = 10; i <= 17; ++i) t.q[17 - i] = (float)(-level(19.0, i) / bottom);  // q[0] = -1 ... q[7]
  t.q[8] = 0.0f;
  for (int i = 9; i <= 15; ++i) t.q[i] = (float)(level(17.0, i) / top);
  for (int j = 0; j < 15; ++j) {
    volatile float sum = t.q[j] + t.q[j + 1];   // one fp32 rounding
    t.m[j] = sum * 0.5f;                        // exact halving
  }
  return t;
}

}  // namespace

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("QL_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

namespace {
struct PerDevice {
  const void* key;
  int tag, dev, val;
};
std::mutex g_pd_mu;
std::vector<PerDevice> g_pd;
}  // namespace

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) {
    cudaGetLastError();
    d = 0;
  }
  return d;
}

int per_device_impl(const void* key, int tag, const std::function<int()>& compute) {
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> g(g_pd_mu);
    for (const PerDevice& e : g_pd)
      if (e.key == key && e.tag == tag && e.dev == dev) return e.val;
  }
  const int v = compute();
  if (v >= 0) {
    std::lock_guard<std::mutex> g(g_pd_mu);
    g_pd.push_back(PerDevice{key, tag, dev, v});   // two first calls may both add the same value
  }
  return v;
}

int device_sm_count() {
  static const int key = 0;
  return per_device(&key, 0, [] {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, current_device()) != cudaSuccess || c <= 0) {
      cudaGetLastError();
      return -1;
    }
    return c;
  });
}

const NF4Table& nf4_table() {
  static NF4Table table = build();
  return table;
}

}  // namespace ql
