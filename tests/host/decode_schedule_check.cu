// Host-side checks of the decode kernel's shared (host and device) schedule
// arithmetic, compiled with nvcc and run on the CPU (no GPU call):
//  - range_lo / range_owner: every item has exactly one owner CTA, whose
//    share holds it, and shares differ by one item at most;
//  - phase-U pieces: the slot run + CTA of each (CTA, run) piece is unique and
//    below runs + CTAs, and walking a run's owners from its first stage
//    (skipping empty shares) finds exactly the pieces that were written;
//  - phase-D shares touch at most two row blocks when D / 128 <= CTAs;
//  - the shared-memory plan fits the opt-in limit with >= 2 ring stages for
//    every supported d_model.
// Prints "OK" and exits 0, or prints the first failure and exits 1.
#include <cstdio>
#include <set>
#include <vector>

#include "../../sparse_moe_ffn_relu_b200/csrc/decode_kernels.cuh"

using namespace deco::dec;

static int fail(const char* what, long a, long b, long c) {
  std::printf("FAIL %s (%ld, %ld, %ld)\n", what, a, b, c);
  return 1;
}

int main() {
  const int Gs[] = {17, 32, 132, 148, 160};
  // shares and owners
  for (int G : Gs)
    for (int n = 1; n <= 5000; n += (n < 300 ? 1 : 97)) {
      int lo_min = 1 << 30, lo_max = 0;
      for (int c = 0; c < G; ++c) {
        const int len = range_lo(c + 1, n, G) - range_lo(c, n, G);
        lo_min = len < lo_min ? len : lo_min;
        lo_max = len > lo_max ? len : lo_max;
      }
      if (lo_max - lo_min > 1) return fail("share sizes", G, n, lo_max - lo_min);
      for (int i = 0; i < n; ++i) {
        const int c = range_owner(i, n, G);
        if (c < 0 || c >= G || range_lo(c, n, G) > i || range_lo(c + 1, n, G) <= i) return fail("owner", G, n, i);
      }
    }
  // phase-U pieces: runs of nkc stages, CTA shares of the stage sequence
  for (int G : Gs)
    for (int nruns : {1, 2, 3, 14, 28, 62, 124, 512})
      for (int nkc : {2, 8, 16, 32}) {
        const int NS = nruns * nkc;
        std::set<int> written;
        for (int c = 0; c < G; ++c) {
          const int s0 = range_lo(c, NS, G), s1 = range_lo(c + 1, NS, G);
          for (int sg = s0; sg < s1; ++sg) {
            const int r = sg / nkc, kc = sg - r * nkc;
            if (kc == nkc - 1 || sg + 1 == s1) {
              const int slot = r + c;
              if (slot >= nruns + G || !written.insert(slot).second) return fail("piece slot", G, nruns, slot);
            }
          }
        }
        std::set<int> read;
        for (int r = 0; r < nruns; ++r) {
          const int end = (r + 1) * nkc;
          int stages = 0;
          for (int cc = range_owner(r * nkc, NS, G); cc >= 0;) {
            read.insert(r + cc);
            const int a = range_lo(cc, NS, G), b = range_lo(cc + 1, NS, G);
            stages += (b < end ? b : end) - (a > r * nkc ? a : r * nkc);
            const int nxt = b;
            cc = nxt < end ? range_owner(nxt, NS, G) : -1;
          }
          if (stages != nkc) return fail("run coverage", G, nruns, r);
        }
        if (read != written) return fail("pieces read != written", G, nruns, nkc);
      }
  // phase-D shares: at most two row blocks of J units each
  for (int G : Gs)
    for (int D = 256; D <= 4096; D += 256) {
      if (D / kDRows > G) continue;
      const int nrb = D / kDRows;
      for (int J : {1, 2, 5, 18, 43, 66, 260}) {
        const int ND = nrb * J;
        for (int c = 0; c < G; ++c) {
          const int v0 = range_lo(c, ND, G), v1 = range_lo(c + 1, ND, G);
          if (v0 < v1 && (v1 - 1) / J - v0 / J > 1) return fail("row blocks per share", G, D, J);
        }
      }
    }
  // shared memory
  for (int D = 256; D <= 4096; D += 256) {
    const SmemPlan p = layer_smem(D);
    if (p.nstages < 2 || p.total + kStaticReserve > (uint32_t)kSmemLimit) return fail("smem plan", D, p.nstages, p.total);
  }
  std::printf("OK\n");
  return 0;
}
