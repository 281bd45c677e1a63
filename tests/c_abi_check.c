/* Compiled as C99 against include/pa.h and linked against libpa.so by the host tests:
 * the header is plain C and every declared entry point resolves.  Run without a GPU, it
 * checks the calls that need no device: pa_version, pa_init's refusal, pa_last_error and
 * the NULL-context checks. */
#include <stdio.h>
#include <string.h>

#include "pa.h"

int main(void) {
  /* every entry point, by address */
  void* fns[] = {(void*)pa_init, (void*)pa_destroy, (void*)pa_last_error, (void*)pa_sync_status,
                 (void*)pa_version, (void*)pa_partition_attn, (void*)pa_merge_states,
                 (void*)pa_compose_states, (void*)pa_merge_states_noalloc, (void*)pa_importance,
                 (void*)pa_state_drift, (void*)pa_selftest_wait, (void*)pa_relayout_seq2head};
  for (size_t i = 0; i < sizeof fns / sizeof fns[0]; ++i)
    if (!fns[i]) return 10;
  const char* v = pa_version();
  if (!v || !strstr(v, "sm_100a")) return 11;
  pa_ctx* ctx = NULL;
  if (pa_init(0, &ctx) == PA_OK) {       /* a B200 is present: nothing more to check here */
    pa_destroy(ctx);
    printf("device present\n");
    return 0;
  }
  if (ctx != NULL) return 12;
  if (!pa_last_error(NULL) || !pa_last_error(NULL)[0]) return 13;
  if (pa_partition_attn(NULL, NULL, NULL) != PA_EINVAL) return 14;
  if (pa_merge_states(NULL, NULL, NULL) != PA_EINVAL) return 15;
  if (pa_selftest_wait(NULL, 0.01, NULL) != PA_EINVAL) return 16;
  pa_attn_desc ad;
  pa_merge_desc md;
  memset(&ad, 0, sizeof ad);
  memset(&md, 0, sizeof md);
  ad.dtype = PA_BF16;
  md.dtype = PA_F32;
  printf("ok: %s\n", v);
  return 0;
}
