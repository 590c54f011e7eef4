/* A plain C99 caller of the library, built and run by tests/test_abi_host.py
 * (no GPU needed): the header compiles as C, the shared library links from C,
 * and its host-side answers -- workspace sizes, argument checks, status
 * strings -- are the ones the Python binding reads.  Prints one "key value"
 * line per answer. */
#include <stdio.h>
#include <string.h>

#include "chunked_kl.h"

static kl_problem topk_problem(void) {
  kl_problem p;
  memset(&p, 0, sizeof p);
  p.N = 4096;
  p.d = 3072;
  p.V = 128256;
  p.dtype = KL_DTYPE_BF16;
  p.teacher = KL_TEACHER_TOPK;
  p.T = 1.0f;
  p.K = 64;
  return p;
}

int main(void) {
  kl_problem p = topk_problem();
  int e;
  printf("sizeof_problem %lu\n", (unsigned long)sizeof(kl_problem));
  for (e = KL_ENTRY_FWD; e <= KL_ENTRY_FWD_BWD; ++e)
    printf("ws_topk_%d %lu\n", e, (unsigned long)kl_workspace_bytes(&p, e));

  p.teacher = KL_TEACHER_HIDDEN;
  p.K = 0;
  p.d_t = 4096;
  p.N = 8192;
  p.T = 2.0f;
  printf("ws_hidden %lu\n", (unsigned long)kl_workspace_bytes(&p, KL_ENTRY_FWD_BWD));

  /* invalid problems: no workspace size, and the calls refuse them before
     touching a device */
  p = topk_problem();
  p.T = 0.0f;
  printf("ws_bad_T %lu\n", (unsigned long)kl_workspace_bytes(&p, KL_ENTRY_FWD_BWD));
  printf("fwd_bwd_bad_T %d\n",
         kl_fwd_bwd(&p, NULL, 0, 1.0f, NULL, NULL, NULL, NULL, 0, NULL));
  p = topk_problem();
  p.d = 3070; /* not a multiple of 8 */
  printf("fwd_bwd_bad_d %d\n",
         kl_fwd_bwd(&p, NULL, 0, 1.0f, NULL, NULL, NULL, NULL, 0, NULL));
  p = topk_problem(); /* H and W are NULL */
  printf("fwd_null_inputs %d\n", kl_fwd(&p, NULL, 0, NULL, NULL, NULL, NULL, NULL));
  printf("fwd_bwd_null %d\n", kl_fwd_bwd(NULL, NULL, 0, 1.0f, NULL, NULL, NULL, NULL, 0, NULL));
  printf("status_string_align %s\n", kl_status_string(KL_ERR_ALIGN));
  printf("noalloc_scratch %lu\n", (unsigned long)KL_NOALLOC_SCRATCH_BYTES);
  return 0;
}
