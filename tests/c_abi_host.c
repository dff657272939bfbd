/*
 * The C ABI used from C: this program includes include/fp8q.h as plain C,
 * links libfp8q.so and exercises the calls that need no device (sizes,
 * status strings, the quantizer pick) and the argument checks that return
 * before anything is launched. Prints "ok" and exits 0 when every check
 * holds; otherwise names the first failure and exits 1.
 */
#include <stdio.h>
#include <string.h>

#include "fp8q.h"

static int failures = 0;

#define CHECK(cond)                                                  \
    do {                                                             \
        if (!(cond)) {                                               \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            failures++;                                              \
        }                                                            \
    } while (0)

int main(void)
{
    /* stand-ins for device pointers: 16-byte aligned, never dereferenced */
    void *a = (void *)0x10000, *b = (void *)0x20000, *c = (void *)0x30000, *d = (void *)0x40000;
    void *odd = (void *)0x10008;
    fp8q_quant_pick_t pick;
    size_t off[6];

    CHECK(fp8q_version() != NULL && strlen(fp8q_version()) > 0);
    CHECK(strncmp(fp8q_status_string(FP8Q_OK), "FP8Q_OK", 7) == 0);
    CHECK(fp8q_status_string((fp8q_status)99) != NULL);
    CHECK(fp8q_m_pad(0) == 0 && fp8q_m_pad(1) == 16 && fp8q_m_pad(16) == 16 && fp8q_m_pad(17) == 32);

    /* the pick keeps kernel and grid together; forcing a variant is reported */
    CHECK(fp8q_quant_pick(4576, 17408, 148, FP8Q_QUANT_AUTO, &pick) == FP8Q_OK);
    CHECK(pick.variant == FP8Q_QUANT_MULTI && pick.forced == 0 && pick.grid_x == pick.multi_ctas);
    CHECK(fp8q_quant_pick(1, 5120, 148, FP8Q_QUANT_AUTO, &pick) == FP8Q_OK && pick.variant == FP8Q_QUANT_SINGLE);
    CHECK(fp8q_quant_pick(1, 5120, 148, FP8Q_QUANT_MULTI, &pick) == FP8Q_OK && pick.forced == 1);
    CHECK(fp8q_quant_pick(1, 100, 148, FP8Q_QUANT_AUTO, &pick) == FP8Q_ERR_SHAPE);
    CHECK(fp8q_quant_pick(1, 5120, 0, FP8Q_QUANT_AUTO, &pick) == FP8Q_ERR_ARG);

    /* workspace sizes */
    CHECK(fp8q_linear_workspace_bytes(17, 512) >= (size_t)17 * 512 + 4 * 4 * 32);
    CHECK(fp8q_ffn_workspace_layout(17, 256, 384, off) == FP8Q_OK && off[0] == 0 && off[5] > off[4]);
    CHECK(fp8q_nvfp4_sf_mma_bytes(129, 5120) == (size_t)256 * 5120 / 16);

    /* argument checks return before any launch */
    CHECK(fp8q_quant_act(a, b, NULL, (float *)c, 4, 100, NULL) == FP8Q_ERR_SHAPE);
    CHECK(fp8q_quant_act(NULL, b, NULL, (float *)c, 4, 128, NULL) == FP8Q_ERR_NULL);
    CHECK(fp8q_quant_act(odd, b, NULL, (float *)c, 4, 128, NULL) == FP8Q_ERR_ALIGN);
    CHECK(fp8q_quant_act(NULL, NULL, NULL, NULL, 0, 128, NULL) == FP8Q_OK);
    CHECK(fp8q_gemm_blockscaled(a, (float *)b, c, (float *)d, a, 4, 100, 128, NULL) == FP8Q_ERR_SHAPE);
    CHECK(fp8q_gemm_ex(a, (float *)b, c, (float *)d, 7, a, 4, 128, 128, NULL) == FP8Q_ERR_ARG);
    CHECK(fp8q_linear(a, b, (float *)c, d, (void *)0x1000010, 1u << 20, 4, 128, 128, NULL) == FP8Q_ERR_WORKSPACE);
    CHECK(fp8q_nvfp4_quant(a, b, NULL, c, 0.0f, 4, 64, NULL) == FP8Q_ERR_ARG);
    CHECK(fp8q_nvfp4_gemm(a, b, 1.0f, c, d, 1.0f, a, 4, 256, 128, NULL) == FP8Q_ERR_SHAPE);
    CHECK(fp8q_dequant_fp8_bf16(a, (float *)b, 2, c, 128, 128, NULL) == FP8Q_ERR_ARG);

    if (failures)
        return 1;
    printf("ok\n");
    return 0;
}
