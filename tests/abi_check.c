/* A plain C11 program against include/tile3d.h and libtile3d.so: the header must compile as C and
 * the host-side calls must work without a GPU. Prints the geometry of the grid given on the command
 * line (B T H W heads D) and the status codes of a few calls that must fail validation. */
#include <stdio.h>
#include <stdlib.h>

#include "tile3d.h"
#include "tile3d_packed.h"

int main(int argc, char** argv) {
  if (argc != 7) {
    fprintf(stderr, "usage: %s B T H W heads D\n", argv[0]);
    return 2;
  }
  t3d_geom g;
  g.B = atoi(argv[1]);
  g.T = atoi(argv[2]);
  g.H = atoi(argv[3]);
  g.W = atoi(argv[4]);
  g.heads = atoi(argv[5]);
  g.D = atoi(argv[6]);
  g.heads_total = 0; /* every head of the row */
  g.head0 = 0;
  int nT = 0, Lp = 0;
  t3d_status st = tile3d_geometry(&g, &nT, &Lp, NULL);
  if (st != T3D_OK) {
    printf("geometry_status %d %s\n", (int)st, t3d_last_error_string());
    return 0;
  }
  int32_t* vc = (int32_t*)malloc(sizeof(int32_t) * (size_t)nT);
  st = tile3d_geometry(&g, &nT, &Lp, vc);
  printf("version %s\n", t3d_version());
  printf("nT %d Lp %d\n", nT, Lp);
  printf("vc");
  for (int i = 0; i < nT; ++i) printf(" %d", vc[i]);
  printf("\n");
  free(vc);
  /* Validation failures, all caught on the host before anything touches a device. */
  printf("scatter_null %d\n", (int)tile3d_scatter(&g, NULL, NULL, NULL));
  printf("topk_k0 %d\n", (int)tile_select_topk(&g, NULL, NULL, 0, NULL, NULL, NULL, 0, NULL, NULL));
  printf("ws_null_geom %zu\n", block_sparse_attn_workspace_size(NULL, 4));
  return 0;
}
