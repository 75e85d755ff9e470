// Host build of the grouped output projection's arithmetic (csrc/out_proj.cuh) for the CPU
// tests: the same split geometry, index functions and per-thread order of the sums (rows
// ascending within a split, splits added in order), on host arrays, with every index checked
// against its buffer. Test infrastructure: the library never links it.
#include <cstdint>
#include <cstring>
#include <vector>

#include "out_proj.cuh"

using namespace csa::proj;

namespace {

float bf(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// one matrix: partial[s][q][col0 + f] = sum over rows of split s of x(q, k) * W(k, f)
template <typename XFn, typename WFn, typename PFn>
int splits(const Geom& G, int K, int ks, int S, int F, XFn x, WFn widx, const uint16_t* W,
           size_t w_elems, PFn pidx, float* part, size_t p_elems) {
  for (int s = 0; s < S; ++s) {
    const int k0 = s * ks, k1 = k0 + ks < K ? k0 + ks : K;
    for (int f0 = 0; f0 < F; f0 += kColsPerThread)
      for (int q = 0; q < G.Q; ++q) {
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int k = k0; k < k1; ++k) {
          const size_t wi = widx(k, f0);
          if (wi + 8 > w_elems) return -1;
          uint4 w;
          memcpy(&w, W + wi, 16);
          float wv[8];
          widen8(w, wv);
          const float xv = x(q, k);
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(xv, wv[i], acc[i]);
        }
        for (int i = 0; i < 8; ++i) {
          const size_t pi = pidx(s, q, f0 + i);
          if (pi >= p_elems) return -2;
          part[pi] = acc[i];
        }
      }
  }
  return 0;
}

}  // namespace

// Returns 0, or a negative code if an index would leave its buffer. geom: S1, S2, ks1, ks2.
extern "C" int out_proj_host(int Q, int H, int c, int g, int d_g, int d, int sms,
                             const uint16_t* o, const uint16_t* w_grp, const uint16_t* w_out,
                             uint16_t* out, int32_t* geom) {
  const Geom G = make_geom(Q, H, c, g, d_g, d, sms);
  geom[0] = G.S1; geom[1] = G.S2; geom[2] = G.ks1; geom[3] = G.ks2;
  std::vector<float> part1(part1_elems(G)), mid(mid_elems(G)), part2(part2_elems(G));
  const size_t o_elems = (size_t)Q * H * c, wg_elems = (size_t)g * G.K1 * d_g;
  const size_t wo_elems = (size_t)g * d_g * d;
  for (int z = 0; z < g; ++z) {
    auto x = [&](int q, int k) {
      const size_t i = o_index(G, q, z, k);
      return i < o_elems ? bf(o[i]) : 1e30f;
    };
    auto widx = [&](int k, int f) { return wgrp_index(G, z, k, f); };
    auto pidx = [&](int s, int q, int f) { return part1_index(G, s, q, z * d_g + f); };
    const int rc = splits(G, G.K1, G.ks1, G.S1, d_g, x, widx, w_grp, wg_elems, pidx,
                          part1.data(), part1.size());
    if (rc) return rc;
  }
  for (int q = 0; q < Q; ++q)
    for (int k = 0; k < g * d_g; ++k) mid[mid_index(G, q, k)] = mid_value(G, part1.data(), q, k);
  auto x2 = [&](int q, int k) { return mid[mid_index(G, q, k)]; };
  auto widx2 = [&](int k, int f) { return wout_index(G, k, f); };
  auto pidx2 = [&](int s, int q, int f) { return part2_index(G, s, q, f); };
  const int rc = splits(G, g * d_g, G.ks2, G.S2, d, x2, widx2, w_out, wo_elems, pidx2,
                        part2.data(), part2.size());
  if (rc) return rc - 10;
  for (int q = 0; q < Q; ++q)
    for (int f = 0; f < d; ++f) {
      const __nv_bfloat16 b = __float2bfloat16_rn(out_value(G, part2.data(), q, f));
      memcpy(&out[(size_t)q * d + f], &b, 2);
    }
  return 0;
}
