/* A plain C99 caller of the library: the header must compile as C, and the
 * host-side entry points (no GPU work) must link and answer. */
#include <stdio.h>

#include "tra.h"

int main(void) {
  tra_grid grid = {21, 45, 80};
  tra_tile tile = {1, 4, 4};
  int s;
  printf("version %d\n", tra_version());
  for (s = TRA_OK; s <= TRA_ERR_BAD_INPUT; ++s) printf("status %d %s\n", s, tra_status_string((tra_status)s));
  printf("workspace %lu\n", (unsigned long)tra_mask_workspace_size(40, grid, tile, 128, 128));
  printf("workspace_bad %lu\n", (unsigned long)tra_mask_workspace_size(40, grid, tile, 96, 128));
  printf("workspace_default_tile %lu\n", (unsigned long)tra_workspace_size(40, grid, 128, 128));
  /* argument checks come before any device work */
  printf("permute_null %d\n", (int)tra_tile_major_permute(NULL, NULL, TRA_BF16, TRA_BF16, 40, 128,
                                                           grid, tile, NULL));
  return 0;
}
