/* c_abi_check.c -- test infrastructure: a plain C99 caller of include/gqe.h.
 * It shows that the header is valid C (no C++ in the ABI), that the library
 * links from C, and that the calls reject bad arguments before touching the
 * GPU.  It makes no call that reaches CUDA, so it runs on a machine without
 * a GPU. */
#include <stdio.h>

#include "gqe.h"

static int fails = 0;
#define EXPECT(c)                                          \
  do {                                                     \
    if (!(c)) {                                            \
      printf("FAILED line %d: %s\n", __LINE__, #c);        \
      ++fails;                                             \
    }                                                      \
  } while (0)

int main(void) {
  /* the main layer: B 8, T 2048, d_model 1024, G 8, E 2, k 1, d_head 64, one shared head */
  gqe_dims d = {8, 2048, 1024, 8, 2, 1, 64, 1, 0, 0, 0.0f, 0};
  gqe_dims chunk = d;
  gqe_layer_weights w = {0};
  size_t whole = 0, host = 0, qproj = 0, oproj = 0;

  EXPECT(gqe_workspace_size(&d, GQE_OP_LAYER_FORWARD, 0, &whole) == GQE_OK);
  EXPECT(gqe_workspace_size(&d, GQE_OP_ROUTED_QPROJ, 0, &qproj) == GQE_OK);
  EXPECT(gqe_workspace_size(&d, GQE_OP_COMBINE_OUT_PROJ, 0, &oproj) == GQE_OK);
  EXPECT(qproj > 0 && oproj > 0 && qproj + oproj < whole);
  chunk.B = 2;
  EXPECT(gqe_workspace_size(&chunk, GQE_OP_LAYER_FORWARD_HOST, 0, &host) == GQE_OK);
  EXPECT(host > 4u * 2u * 2048u * 1024u * 2u);      /* two x and two y chunk buffers at least */

  /* argument errors come back before any launch */
  EXPECT(gqe_layer_forward(&d, NULL, NULL, NULL, NULL, 0, NULL) == GQE_ERR_INVALID_ARG);
  EXPECT(gqe_layer_forward_host(&d, &w, NULL, NULL, 2, NULL, 0, NULL, NULL, NULL) == GQE_ERR_INVALID_ARG);
  EXPECT(gqe_router_topk(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == GQE_ERR_INVALID_ARG);
  d.d_head = 96;
  EXPECT(gqe_workspace_size(&d, GQE_OP_LAYER_FORWARD, 0, &whole) == GQE_ERR_UNSUPPORTED);
  EXPECT(gqe_status_string(GQE_ERR_WORKSPACE)[0] != '\0');

  printf("%s\n", fails ? "c-abi: failures" : "c-abi: ok");
  return fails != 0;
}
