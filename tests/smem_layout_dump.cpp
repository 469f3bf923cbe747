// Prints fb_smem_layout for every team shape the bitshift launches can take,
// with the staging decision the host makes (fb_xstage), one line per case:
//   L k adj alias nseq cluster NT tpc GL NV xstage exA exF exB exBt mbar per_seq per_team red
//   stage stageF stageK xst xstF cf total
// Built and run on the CPU by tests/test_smem_layout.py.
#include <cstdio>

#include "bcjr_internal.h"

int main() {
  for (int L = 4; L <= 16; ++L) {
    const int TS = (1 << L) / 16;  // 16 states per thread
    int NT, cluster, tpc;
    if (TS > 512) {
      NT = 512;
      cluster = TS / 512;
      tpc = 1;
    } else if (TS >= 32) {
      NT = TS;
      cluster = 1;
      tpc = 1;
    } else {
      NT = 32;
      cluster = 1;
      tpc = 32 / TS;
    }
    for (int k = 1; k <= 4 && k <= L; ++k) {
      const int K = 1 << k;
      const int NV = (K <= 4 ? 16 / (K * K) : 1) * (K < 4 ? K : 4);
      const int GL = ((1 << L) >> k) / cluster;
      for (int adj = 0; adj <= 1; ++adj)
        for (int alias = 0; alias <= 1; ++alias) {
          const int base = (cluster > 1 && k >= 2) ? 2 : 1;
          const int top = (base == 2 && !adj) ? 4 : base;  // the forward call may ask for 3 or 4
          for (int nseq = base; nseq <= top; ++nseq) {
            const bool xs = bcjr::fb_xstage(cluster, k, nseq, adj != 0, alias != 0);
            const bcjr::FBSmem l = bcjr::fb_smem_layout(GL, NT, NV, nseq, adj != 0, alias != 0, tpc, xs);
            std::printf("%d %d %d %d %d %d %d %d %d %d %d %u %u %u %u %u %u %u %u %u %u %u %u %u %u %u\n", L, k, adj,
                        alias, nseq, cluster, NT, tpc, GL, NV, xs ? 1 : 0, l.exA, l.exF, l.exB, l.exBt, l.mbar,
                        l.per_seq, l.per_team, l.red, l.stage, l.stageF, l.stageK, l.xst, l.xstF, l.cf, l.total);
          }
        }
    }
  }
  return 0;
}
