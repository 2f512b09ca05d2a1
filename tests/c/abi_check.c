/* A plain C99 caller of libnf4lora: compiles against include/nf4lora.h alone
 * (no C++ and no CUDA headers) and exercises the host-only entry points --
 * sizing, buffer layout and argument checks that return before any device
 * work -- so it runs without a GPU.  Prints "ok" and exits 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "nf4lora.h"

#define CHECK(cond)                                                             \
    do {                                                                        \
        if (!(cond)) {                                                          \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            return 1;                                                           \
        }                                                                       \
    } while (0)

int main(void) {
    const int64_t d_out = 4096, d_in = 4096, n = d_out * d_in;
    /* storage: n/2 code bytes + n/64 int8 scales + 4 n/16384 + 4, each part padded to 256 */
    const size_t bytes = nf4_packed_bytes(d_out, d_in);
    CHECK(bytes >= (size_t)(n / 2 + n / 64 + 4 * (n / 16384) + 4));
    CHECK(bytes < (size_t)(n / 2 + n / 64 + 4 * (n / 16384) + 4 + 4 * 256));
    CHECK(nf4_packed_bytes(4096, 100) == 0); /* d_in % 64 != 0 */

    nf4_tensor t;
    memset(&t, 0, sizeof t);
    uintptr_t base = (uintptr_t)1 << 20; /* never dereferenced on the host */
    CHECK(nf4_tensor_from_buffer(&t, (void*)base, bytes, d_out, d_in) == NF4_OK);
    CHECK((uintptr_t)t.codes == base);
    CHECK((uintptr_t)t.qscale - (uintptr_t)t.codes >= (uintptr_t)(n / 2));
    CHECK(((uintptr_t)t.qscale & 255u) == 0 && ((uintptr_t)t.scale2 & 255u) == 0);
    CHECK(nf4_tensor_from_buffer(&t, (void*)base, bytes - 1, d_out, d_in) != NF4_OK);

    CHECK(t.absmax == NULL); /* the double-quantised format */

    /* fp32 block scales (no double quantisation): n/2 + 4 n/64 bytes, each part padded to 256 */
    const size_t bytes_nodq = nf4_packed_bytes_nodq(d_out, d_in);
    CHECK(bytes_nodq >= (size_t)(n / 2 + 4 * (n / 64)));
    CHECK(bytes_nodq < (size_t)(n / 2 + 4 * (n / 64) + 2 * 256));
    CHECK(nf4_packed_bytes_nodq(4096, 100) == 0);
    nf4_tensor u;
    memset(&u, 0xff, sizeof u);
    CHECK(nf4_tensor_from_buffer_nodq(&u, (void*)base, bytes_nodq, d_out, d_in) == NF4_OK);
    CHECK((uintptr_t)u.codes == base && u.qscale == NULL && u.scale2 == NULL && u.scale_mean == NULL);
    CHECK((uintptr_t)u.absmax - base >= (uintptr_t)(n / 2) && ((uintptr_t)u.absmax & 255u) == 0);
    CHECK(nf4_tensor_from_buffer_nodq(&u, (void*)base, bytes_nodq - 1, d_out, d_in) != NF4_OK);

    CHECK(nf4_quantize_workspace_bytes(d_out, d_in) > 0);
    CHECK(qlora_fwd_workspace_bytes(16, d_out, d_in, 64) > 0);
    CHECK(qlora_bwd_workspace_bytes(4096, d_out, d_in, 64) > qlora_bwd_workspace_bytes(16, d_out, d_in, 64));
    CHECK(nf4_merge_workspace_bytes(d_out, d_in) >= (size_t)(4 * n));

    /* argument checks return a status and enqueue nothing */
    const uint16_t* A = (const uint16_t*)((uintptr_t)1 << 24);
    const uint16_t* B = (const uint16_t*)((uintptr_t)1 << 25);
    uint16_t* Y = (uint16_t*)((uintptr_t)1 << 27);
    CHECK(qlora_linear_fwd(&t, A, B, 64, 0.25f, NULL, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_INVALID_ARG);
    CHECK(qlora_linear_fwd(&t, A, B, 0, 0.25f, Y, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_INVALID_ARG);   /* r < 1 */
    CHECK(qlora_linear_fwd(&t, A, B, 257, 0.25f, Y, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_INVALID_ARG); /* r > 256 */
    /* any rank in [1, 256]: r = 12 passes the argument checks and needs a workspace */
    CHECK(qlora_linear_fwd(&t, A, B, 12, 0.25f, Y, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_WORKSPACE);
    CHECK(qlora_fwd_workspace_bytes(16, d_out, d_in, 12) > qlora_fwd_workspace_bytes(16, d_out, d_in, 16));
    CHECK(strlen(nf4lora_last_error_string()) > 0);
    CHECK(qlora_linear_fwd(&t, A, B, 64, 0.25f, NULL, 0, NULL, NULL, NULL, 0, NULL) == NF4_OK); /* empty batch */
    CHECK(nf4_merge_lora(&t, A, B, 0, 1.0f, (float*)Y, NULL) == NF4_ERR_INVALID_ARG);
    CHECK(qlora_linear_fwd(&u, A, B, 64, 0.25f, NULL, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_INVALID_ARG);
    u.codes = NULL;
    CHECK(qlora_linear_fwd(&u, A, B, 64, 0.25f, Y, 16, Y, NULL, NULL, 0, NULL) == NF4_ERR_INVALID_ARG);

    lora_adamw_tensor at;
    memset(&at, 0, sizeof at);
    lora_adamw_hparams hp = {1e-3f, 0.9f, 0.999f, 1e-8f, 0.0f, 0};
    CHECK(lora_adamw_step(&at, 1, &hp, NULL) == NF4_ERR_INVALID_ARG); /* step counts from 1 */

    CHECK(strstr(nf4lora_version(), "sm_100a") != NULL);
    printf("ok\n");
    return 0;
}
