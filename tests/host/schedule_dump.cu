// Host-only program: prints the query-group schedule of the CUDA path for a
// layout given on the command line, one group per line, so that the test suite
// can check it against the oracle's key sets on the CPU (no GPU needed).
#include <cstdio>
#include <cstdlib>

#include "../../linear_attention_video_block_b200/csrc/vdn_internal.cuh"

int main(int argc, char** argv) {
  if (argc != 5 && argc != 8) {
    std::fprintf(stderr, "usage: schedule_dump F N c rows [T A ctx]\n");
    return 2;
  }
  vdn::Layout l;
  l.B = 1; l.H = 1; l.d = 16; l.T = 1;
  l.F = std::atoi(argv[1]); l.N = std::atoi(argv[2]); l.c = std::atoi(argv[3]);
  const int rows = std::atoi(argv[4]);
  if (argc == 8) { l.T = std::atoi(argv[5]); l.A = std::atoi(argv[6]); l.ctx = std::atoi(argv[7]); }
  int fwd_max, rev_min;
  vdn::scan_extent(l, fwd_max, rev_min);
  std::printf("extent %d %d tiles %d\n", fwd_max, rev_min, vdn::tiles_per_head(l, rows));
  for (int g = 0; g < l.groups(); ++g) {
    vdn::Group G = vdn::make_group(l, g);
    std::printf("group %d q0 %d nq %d chunk %d fwd %d rev %d segs", g, G.q0, G.nq, G.chunk,
                G.fwd_idx, G.rev_idx);
    for (int s = 0; s < G.nseg; ++s) std::printf(" %d:%d", G.seg0[s], G.segn[s]);
    std::printf("\n");
    std::printf("qsrc %d %d\n", g, G.qsrc);
  }
  for (int g = 0; g < l.groups(); ++g) {
    vdn::Group G = vdn::make_group(l, g);
    if (G.nq == 0) continue;
    const int nk = vdn::key_tile_count(G, l.T, l.A, 128);
    std::printf("keytiles %d", g);
    for (int t = 0; t < nk; ++t) {
      vdn::KeyTile k = vdn::key_tile(G, l.T, l.A, t, 128);
      std::printf(" %d:%d:%d", k.src, k.row, k.valid);
    }
    std::printf("\n");
  }
  const int nt = vdn::tiles_per_head(l, rows);
  for (int t = 0; t < nt; ++t) {
    int g, r0;
    vdn::tile_to_group(l, rows, t, g, r0);
    std::printf("tile %d group %d r0 %d\n", t, g, r0);
  }
  return 0;
}
