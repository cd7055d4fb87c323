/* Uses the C ABI from plain C on a GPU (no Python, no PyTorch): cudaMalloc'd
 * buffers, three opt2s_step calls and two opt2s_step_max_unorm calls on a
 * mixed fp32/fp16/bf16 AdEMAMix collection with a misaligned tensor, then a
 * bitwise comparison with the CPU oracle (test infrastructure, linked only
 * into this test).  Built and run by tests/test_c_abi.py.  Prints "ok" on
 * success. */
#include <stdio.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "opt2s.h"

int oracle_step_f32(int algo, int dtype, int skip_zeros, float lr, float beta1, float beta2,
                    float beta3, float alpha, float eps, float weight_decay, int step,
                    void *param, const void *grad, float *state1, float *state2, int64_t n);
int oracle_step_f32_max_unorm(int algo, int dtype, int skip_zeros, float lr, float beta1,
                              float beta2, float beta3, float alpha, float eps,
                              float weight_decay, float max_unorm, int step, void *param,
                              const void *grad, float *state1, float *state2, int64_t n,
                              float *scale_out);
uint16_t oracle_f32_to_f16(float x);
uint16_t oracle_f32_to_bf16(float x);

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { printf("CUDA %d at line %d\n", (int)e_, __LINE__); return 1; } } while (0)

static uint64_t state = 0x0E0A0000ull;
static float next_uniform(void)   /* SplitMix64 output function on a counter */
{
    uint64_t z = (state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    return (float)((z >> 40) * (1.0 / 16777216.0)) * 2.0f - 1.0f;
}

int main(void)
{
    enum { T = 3 };
    const int64_t n[T] = {1000, 4097, 33};
    const int dt[T] = {OPT2S_F32, OPT2S_F16, OPT2S_BF16};
    const int offset[T] = {0, 0, 1};          /* tensor 2 starts one element in */
    Hyper h = {2e-3f, 0.9f, 0.999f, 0.99f, 5.0f, 1e-8f, 0.1f, OPT2S_ADEMAMIX, 0};
    opt2s_tensor rec[T];
    void *hp[T], *hg[T], *dp[T], *dg[T];
    float *hs1[T], *hs2[T], *ds1[T], *ds2[T];
    for (int i = 0; i < T; ++i) {
        const int es = dt[i] == OPT2S_F32 ? 4 : 2;
        const size_t bytes = (size_t)(n[i] + offset[i]) * es;
        hp[i] = calloc(n[i] + offset[i], es);
        hg[i] = calloc(n[i] + offset[i], es);
        hs1[i] = calloc(2 * n[i], 4);
        hs2[i] = calloc(n[i], 4);
        for (int64_t k = 0; k < n[i]; ++k) {
            float p = next_uniform(), g = next_uniform() * 1e-2f;
            char *P = (char *)hp[i] + (k + offset[i]) * es, *G = (char *)hg[i] + (k + offset[i]) * es;
            if (dt[i] == OPT2S_F32) { memcpy(P, &p, 4); memcpy(G, &g, 4); }
            else {
                uint16_t a = dt[i] == OPT2S_F16 ? oracle_f32_to_f16(p) : oracle_f32_to_bf16(p);
                uint16_t b = dt[i] == OPT2S_F16 ? oracle_f32_to_f16(g) : oracle_f32_to_bf16(g);
                memcpy(P, &a, 2); memcpy(G, &b, 2);
            }
        }
        CK(cudaMalloc(&dp[i], bytes));
        CK(cudaMalloc(&dg[i], bytes));
        CK(cudaMalloc((void **)&ds1[i], 8 * n[i]));
        CK(cudaMalloc((void **)&ds2[i], 4 * n[i]));
        CK(cudaMemcpy(dp[i], hp[i], bytes, cudaMemcpyHostToDevice));
        CK(cudaMemcpy(dg[i], hg[i], bytes, cudaMemcpyHostToDevice));
        CK(cudaMemset(ds1[i], 0, 8 * n[i]));
        CK(cudaMemset(ds2[i], 0, 4 * n[i]));
        rec[i].param = (char *)dp[i] + offset[i] * es;
        rec[i].grad = (const char *)dg[i] + offset[i] * es;
        rec[i].state1 = ds1[i];
        rec[i].state2 = ds2[i];
        rec[i].numel = n[i];
        rec[i].dtype = dt[i];
        rec[i].reserved = 0;
    }
    TensorListDesc d = {rec, T};
    const float max_unorm = 0.05f;           /* steps 4 and 5: bounded update norm */
    for (int step = 1; step <= 5; ++step) {
        int st = step <= 3 ? opt2s_step(&d, &h, step, 0)
                           : opt2s_step_max_unorm(&d, &h, max_unorm, step, 0);
        if (st != OPT2S_OK) { printf("step %d: %s\n", step, opt2s_error_string(st)); return 1; }
        for (int i = 0; i < T; ++i) {
            const int es = dt[i] == OPT2S_F32 ? 4 : 2;
            if (step <= 3)
                oracle_step_f32(1, dt[i], 0, h.lr, h.beta1, h.beta2, h.beta3, h.alpha, h.eps,
                                h.weight_decay, step, (char *)hp[i] + offset[i] * es,
                                (const char *)hg[i] + offset[i] * es, hs1[i], hs2[i], n[i]);
            else
                oracle_step_f32_max_unorm(1, dt[i], 0, h.lr, h.beta1, h.beta2, h.beta3, h.alpha,
                                          h.eps, h.weight_decay, max_unorm, step,
                                          (char *)hp[i] + offset[i] * es,
                                          (const char *)hg[i] + offset[i] * es, hs1[i], hs2[i],
                                          n[i], NULL);
        }
    }
    CK(cudaDeviceSynchronize());
    for (int i = 0; i < T; ++i) {
        const int es = dt[i] == OPT2S_F32 ? 4 : 2;
        const size_t bytes = (size_t)(n[i] + offset[i]) * es;
        void *gp = malloc(bytes), *gg = malloc(bytes);
        float *g1 = malloc(8 * n[i]), *g2 = malloc(4 * n[i]);
        CK(cudaMemcpy(gp, dp[i], bytes, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(gg, dg[i], bytes, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(g1, ds1[i], 8 * n[i], cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(g2, ds2[i], 4 * n[i], cudaMemcpyDeviceToHost));
        if (memcmp(gp, hp[i], bytes) || memcmp(gg, hg[i], bytes) ||
            memcmp(g1, hs1[i], 8 * n[i]) || memcmp(g2, hs2[i], 4 * n[i])) {
            printf("FAIL: tensor %d differs from the oracle\n", i);
            return 1;
        }
        free(gp); free(gg); free(g1); free(g2);
        cudaFree(dp[i]); cudaFree(dg[i]); cudaFree(ds1[i]); cudaFree(ds2[i]);
    }
    opt2s_release_cache();
    printf("ok\n");
    return 0;
}
