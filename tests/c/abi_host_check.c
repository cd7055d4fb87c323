/* Uses the C ABI from plain C, without a GPU: argument validation and error
 * codes.  Built and run by tests/test_c_abi.py.  Prints "ok" on success. */
#include <stdio.h>
#include <stdint.h>
#include "opt2s_testing.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void)
{
    CHECK(opt2s_abi_version() == OPT2S_ABI_VERSION);
    opt2s_tensor t = {(void *)0x10000000, (const void *)0x20000000, (float *)0x30000000,
                      (float *)0x40000000, 1024, OPT2S_F32, 0};
    TensorListDesc d = {&t, 1};
    Hyper h = {1e-3f, 0.9f, 0.999f, 0.0f, 0.0f, 1e-8f, 0.0f, OPT2S_ADAM, 0};
    CHECK(opt2s_testing_validate(&d, &h, 1) == OPT2S_OK);
    CHECK(opt2s_testing_validate(&d, &h, 0) == OPT2S_ERR_INVALID_ARG);
    CHECK(opt2s_testing_validate(NULL, &h, 1) == OPT2S_ERR_INVALID_ARG);
    CHECK(opt2s_testing_validate(&d, NULL, 1) == OPT2S_ERR_INVALID_ARG);
    t.grad = t.param;
    CHECK(opt2s_testing_validate(&d, &h, 1) == OPT2S_ERR_ALIAS);
    t.grad = (const void *)0x20000000;
    h.beta2 = 1.0f;
    CHECK(opt2s_step(&d, &h, 1, 0) == OPT2S_ERR_INVALID_ARG);   /* no CUDA call reached */
    h.beta2 = 0.999f;
    opt2s_testing_chunk chunks[8];
    int64_t n = 0;
    CHECK(opt2s_testing_build_chunks(&d, OPT2S_ADAM, 256, chunks, 8, &n) == OPT2S_OK && n == 4);
    CHECK(chunks[3].start == 768 && chunks[3].len == 256 && chunks[3].tensor == 0);
    opt2s_step_scalars sc[2];
    CHECK(opt2s_fill_step_scalars(&h, 1, 2, sc) == OPT2S_OK);
    CHECK(sc[0].bc1 == (float)(1.0 - 0.8999999761581421) && sc[1].decay == 1.0f);
    CHECK(opt2s_noalloc_max_chunks() == 65536);
    printf("ok\n");
    return 0;
}
