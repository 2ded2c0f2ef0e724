// Host-side check of the GEMV work split the engine plans (compiled and run
// by tests/test_geometry.py; no GPU needed).  For the decode GEMVs of the
// OLMo-3-32B shape and of the small decoder, at several batch sizes and SM
// counts: the CTA ranges cover the units once and in order, a CTA's units
// span at most two k-slabs and its x range fits shared memory, whole-segment
// modes start and end CTAs on segment boundaries and slab-aligned groups stay
// in their slab.
#include <cstdio>
#include "engine.cuh"
using namespace w4a;

static int fails = 0;
#define CHECK(c, ...)                               \
  do {                                              \
    if (!(c)) {                                     \
      if (++fails <= 20) {                          \
        printf("FAIL line %d: ", __LINE__);         \
        printf(__VA_ARGS__);                        \
        printf("\n");                               \
      }                                             \
    }                                               \
  } while (0)

static void check(const char* name, long long n, long long k, int kcw, int B, int nc, int readers) {
  const int nb = B <= 8 ? 1 : 2;
  const Geo g = gemv_geo(n, k, kcw, B, nb, nc, readers);
  CHECK(g.ns > 0 && g.kps > 0 && g.nca > 0, "%s B %d nc %d: no geometry", name, B, nc);
  if (g.ns <= 0 || g.kps <= 0 || g.nca <= 0) return;
  CHECK(g.ns * g.kps == g.nkc, "%s: slabs x k-chunks %d x %d != %d", name, g.ns, g.kps, g.nkc);
  CHECK(g.nca <= nc, "%s: %d CTAs > %d", name, g.nca, nc);
  const long long U = (long long)g.ns * g.nrb * g.kps, upsl = (long long)g.nrb * g.kps;
  long long prev = 0;
  for (int c = 0; c < nc; ++c) {
    int a, b;
    gemv_cta_range(g, c, a, b);
    if (c >= g.nca) {
      CHECK(a == b, "%s: idle CTA %d has units", name, c);
      continue;
    }
    CHECK(a == prev && b >= a, "%s B %d: CTA %d range [%d, %d) after %lld", name, B, c, a, b, prev);
    prev = b;
    if (a == b) continue;
    CHECK(a % g.kps == 0 && b % g.kps == 0, "%s: CTA %d cuts a segment", name, c);
    const long long s0 = a / upsl, s1 = (b - 1) / upsl;
    CHECK(s1 - s0 <= 1, "%s: CTA %d spans %lld slabs", name, c, s1 - s0 + 1);
    if (g.aligned) CHECK(s0 == s1, "%s: aligned CTA %d spans two slabs", name, c);
    CHECK(x_fits((s1 - s0 + 1) * (long long)g.kps * kcw, B, nb), "%s B %d: CTA %d x range too large", name, B, c);
  }
  CHECK(prev == U, "%s: ranges end at %lld of %lld units", name, prev, U);
}

int main() {
  const int batches[] = {1, 2, 4, 8, 9, 16};
  const int sms[] = {148, 132};
  for (int B : batches)
    for (int nc : sms) {
      // OLMo-3-32B shape: QKV, O, gate/up, down, lm_head
      check("qkv", 7168, 5120, W4_KC, B, nc, nc);
      check("o", 5120, 5120, W4_KC, B, nc, nc);
      check("gate_up", 55296, 5120, W4_KC, B, nc, nc);
      check("down", 5120, 27648, W4_KC, B, nc, nc);
      check("lm_head", 100288, 5120, BF_KC, B, nc, 1);
      // the small decoder
      check("t_qkv", 768, 512, W4_KC, B, nc, nc);
      check("t_o", 512, 512, W4_KC, B, nc, nc);
      check("t_gate_up", 3072, 512, W4_KC, B, nc, nc);
      check("t_down", 512, 1536, W4_KC, B, nc, nc);
      check("t_lm_head", 4096, 512, BF_KC, B, nc, 1);
    }
  printf(fails ? "FAILURES %d\n" : "geometry ok\n", fails);
  return fails ? 1 : 0;
}
