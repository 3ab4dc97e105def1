// pld.cu — Progressive Layer Dropping decisions for a stack of encoder
// layers (host code).
//
// "Progressive Layer Dropping" page, schedule section: the keep level falls
// from 1 towards a target theta_bar as the global step t grows,
//   theta(t) = (1 - theta_bar) * exp(-gamma * t) + theta_bar,
// and layers are skipped at random, more often the deeper they sit.  The
// depth profile, which the page leaves open, is read as linear: layer l of
// L (0-based) is kept with probability 1 - (l + 1) / L * (1 - theta(t)), so
// the first layer is almost always kept and the last with probability
// theta(t).  A skipped layer is the identity in forward and backward.
//
// The random draw uses the Philox4x32-10 stream of the dropout contract with
// site 3: counter (t mod 2^32, t div 2^32, 3, l), key (seed mod 2^32,
// seed div 2^32); layer l is kept when output word 0, read as a 32-bit
// unsigned integer, is below floor(keep_probability * 2^32).  Every rank of
// a data-parallel job that shares the seed and step takes the same
// decisions without communicating.
#include <cmath>
#include <cstdint>

#include "tlp.h"

namespace {

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11), host form.
void philox4x32_10_host(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1;
    c[1] = (uint32_t)p1;
    c[3] = (uint32_t)p0;
    c[0] = n0;
    c[2] = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

constexpr uint32_t kPldSite = 3;

}  // namespace

extern "C" {

double tl_pld_theta(double theta_bar, double gamma, uint64_t step) {
  return (1.0 - theta_bar) * std::exp(-gamma * (double)step) + theta_bar;
}

double tl_pld_keep_prob(int layer, int num_layers, double theta) {
  if (num_layers <= 0 || layer < 0 || layer >= num_layers) return -1.0;
  return 1.0 - (double)(layer + 1) / (double)num_layers * (1.0 - theta);
}

int tl_pld_keep(uint64_t seed, uint64_t step, int layer, int num_layers, double theta) {
  const double p = tl_pld_keep_prob(layer, num_layers, theta);
  if (p < 0.0) return -1;
  if (p >= 1.0) return 1;
  if (!(p > 0.0)) return 0;
  const uint32_t thr = (uint32_t)std::floor(p * 4294967296.0);   // p < 1, so thr < 2^32
  uint32_t c[4] = {(uint32_t)step, (uint32_t)(step >> 32), kPldSite, (uint32_t)layer};
  philox4x32_10_host(c, (uint32_t)seed, (uint32_t)(seed >> 32));
  return c[0] < thr ? 1 : 0;
}

}  // extern "C"
