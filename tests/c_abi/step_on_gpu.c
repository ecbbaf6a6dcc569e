/* One training step through the C ABI from plain C, with device memory from
 * the CUDA runtime and no Python in the process: llm_init draws the
 * parameters, llm_step runs on the legacy default stream, and the parameters
 * before and after, the token and target ids and the loss go to a binary file
 * (argv[1]) for the test that runs the same step in the float64 oracle. */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

#include "llm.h"

#define B 2
#define T 16

static int fail(const char *what, int rc) {
  fprintf(stderr, "%s failed: %d\n", what, rc);
  return 1;
}

int main(int argc, char **argv) {
  if (argc != 2) return fail("usage", 0);
  llm_config c = {.vocab = 27, .d_model = 16, .n_layer = 1, .n_head = 4, .n_kv_head = 2,
                  .d_ff = 42, .ctx = T, .batch = B, .rope_base = 10000.f, .rms_eps = 1e-5f,
                  .beta1 = 0.9f, .beta2 = 0.999f, .adam_eps = 1e-8f, .compute = LLM_FP32,
                  .recompute = 0};
  int n = 0, rc;
  int64_t np = 0, ws = 0;
  if ((rc = llm_param_layout(&c, NULL, &n, &np)) != LLM_OK) return fail("layout", rc);
  if ((rc = llm_workspace_bytes(&c, &ws)) != LLM_OK) return fail("workspace", rc);
  int32_t tok[B * T], tgt[B * T];
  for (int i = 0; i < B * T; i++) {
    tok[i] = (7 * i + 3) % c.vocab;
    tgt[i] = (5 * i + 1) % c.vocab;
  }
  void *dws = NULL;
  float *dp = NULL, *dg = NULL, *dm = NULL, *dv = NULL, *dloss = NULL;
  int32_t *dtok = NULL, *dtgt = NULL;
  const size_t pb = (size_t)np * sizeof(float);
  if (cudaMalloc(&dws, (size_t)ws) || cudaMalloc((void **)&dp, pb) ||
      cudaMalloc((void **)&dg, pb) || cudaMalloc((void **)&dm, pb) ||
      cudaMalloc((void **)&dv, pb) || cudaMalloc((void **)&dloss, sizeof(float)) ||
      cudaMalloc((void **)&dtok, sizeof tok) || cudaMalloc((void **)&dtgt, sizeof tgt))
    return fail("cudaMalloc", 0);
  if (cudaMemset(dm, 0, pb) || cudaMemset(dv, 0, pb) ||
      cudaMemcpy(dtok, tok, sizeof tok, cudaMemcpyHostToDevice) ||
      cudaMemcpy(dtgt, tgt, sizeof tgt, cudaMemcpyHostToDevice))
    return fail("cudaMemcpy", 0);
  llm_ctx *ctx = NULL;
  if ((rc = llm_create(&c, dws, ws, NULL, &ctx)) != LLM_OK) return fail("llm_create", rc);
  if ((rc = llm_init(ctx, 1234, 0.08f, 0, dp)) != LLM_OK) return fail("llm_init", rc);
  float *before = malloc(pb), *after = malloc(pb), loss = 0.f;
  if (!before || !after) return fail("malloc", 0);
  if (cudaMemcpy(before, dp, pb, cudaMemcpyDeviceToHost)) return fail("copy params", 0);
  if ((rc = llm_step(ctx, dp, dg, dm, dv, 1, dtok, dtgt, 1e-2f, 0.1f, dloss)) != LLM_OK)
    return fail("llm_step", rc);
  if ((rc = llm_status(ctx)) != LLM_OK) return fail("llm_status", rc);
  if (cudaMemcpy(after, dp, pb, cudaMemcpyDeviceToHost) ||
      cudaMemcpy(&loss, dloss, sizeof loss, cudaMemcpyDeviceToHost))
    return fail("copy results", 0);
  FILE *f = fopen(argv[1], "wb");
  if (!f) return fail("fopen", 0);
  const int64_t hdr[2] = {np, B * T};
  fwrite(hdr, sizeof hdr, 1, f);
  fwrite(tok, sizeof tok, 1, f);
  fwrite(tgt, sizeof tgt, 1, f);
  fwrite(&loss, sizeof loss, 1, f);
  fwrite(before, pb, 1, f);
  fwrite(after, pb, 1, f);
  fclose(f);
  llm_destroy(ctx);
  cudaFree(dws); cudaFree(dp); cudaFree(dg); cudaFree(dm); cudaFree(dv);
  cudaFree(dloss); cudaFree(dtok); cudaFree(dtgt);
  free(before); free(after);
  printf("loss %.9g\n", loss);
  return 0;
}
