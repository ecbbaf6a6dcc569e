/* A plain C consumer of the library's host-only entry points (no device is
 * touched): the parameter layout and count, the workspace size, the
 * learning-rate schedule, the plateau rule and the gradient buckets of a small
 * GQA config, printed one fact per line for the test that compiles and runs
 * this file. */
#include <stdio.h>

#include "llm.h"

int main(void) {
  llm_config c = {.vocab = 27, .d_model = 16, .n_layer = 2, .n_head = 4, .n_kv_head = 2,
                  .d_ff = 42, .ctx = 16, .batch = 2, .rope_base = 10000.f, .rms_eps = 1e-5f,
                  .beta1 = 0.9f, .beta2 = 0.999f, .adam_eps = 1e-8f, .compute = LLM_FP32,
                  .recompute = 0};
  int n = 0;
  int64_t n_params = 0, ws = 0;
  if (llm_param_layout(&c, NULL, &n, &n_params) != LLM_OK) return 1;
  llm_tensor_info info[64];
  int cap = 64;
  if (n > cap || llm_param_layout(&c, info, &cap, &n_params) != LLM_OK) return 2;
  printf("tensors %d\nparams %lld\n", n, (long long)n_params);
  for (int i = 0; i < n; i++)
    printf("tensor %s %lld %lld %lld\n", info[i].name, (long long)info[i].offset,
           (long long)info[i].rows, (long long)info[i].cols);
  if (llm_workspace_bytes(&c, &ws) != LLM_OK || ws <= 0) return 3;
  printf("workspace %lld\n", (long long)ws);

  llm_lr_schedule sc = {.max_lr = 3e-4f, .min_lr = 3e-5f, .warmup_steps = 10,
                        .decay_start = 10, .total_steps = 110, .shape = LLM_LR_COSINE};
  for (int64_t t = 1; t <= 120; t += 17) {
    float lr = 0.f;
    if (llm_lr_at(&sc, t, &lr) != LLM_OK) return 4;
    printf("lr %lld %.9g\n", (long long)t, lr);
  }

  llm_plateau pl;
  float scale = 0.f;
  if (llm_plateau_init(&pl, 0.5f, 2, 3, 0.0) != LLM_OK) return 5;
  const double metric[10] = {3.0, 2.5, 2.6, 2.6, 2.6, 2.4, 2.4, 2.4, 2.4, 2.4};
  for (int i = 0; i < 10; i++) {
    if (llm_plateau_update(&pl, metric[i], &scale) != LLM_OK) return 6;
    printf("plateau %d %.9g\n", i, scale);
  }

  for (int k = 0; k < c.n_layer + 2; k++) {
    int64_t off = 0, cnt = 0;
    if (llm_grad_bucket_range(&c, k, &off, &cnt) != LLM_OK) return 7;
    printf("bucket %d %lld %lld\n", k, (long long)off, (long long)cnt);
  }
  /* a null context is refused without a device */
  if (llm_forward(NULL, NULL, NULL, NULL) != LLM_ERR_ARG) return 8;
  printf("%s\n", llm_error_string(LLM_ERR_TOKEN));
  return 0;
}
