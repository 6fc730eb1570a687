/* abi_host_check.c -- the C ABI of libsbl.so used from plain C99, with no
 * CUDA header and no device: buffer sizes, the format rule, status strings,
 * and the argument checks that every entry point makes before it looks up
 * a device.  Pointers are fake (never dereferenced: every call below is
 * rejected, or is a no-op, before any device access).
 *
 * Usage: abi_host_check
 * When the library itself reports that no sm_100 device is present
 * (sbl_device_error returns SBL_ERR_DEVICE), valid calls are also checked
 * to report SBL_ERR_DEVICE and enqueue nothing; with a device present those
 * calls are skipped, so no fake pointer ever reaches a kernel.
 * Exit status 0 when every check holds; each failure is printed.          */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "sbl.h"

static int failures = 0;

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                    \
        }                                                                  \
    } while (0)

static size_t round16(size_t x) { return (x + 15) / 16 * 16; }

int main(void)
{
    uint32_t code = 0;
    const int no_device = sbl_device_error(&code, 0) == SBL_ERR_DEVICE;
    /* fake, 16-byte aligned device addresses and a misaligned one */
    void *const A = (void *)(uintptr_t)0x100000;
    void *const B = (void *)(uintptr_t)0x200000;
    void *const MIS = (void *)(uintptr_t)0x300008;

    CHECK(sbl_version() > 0);
    for (int s = SBL_OK; s <= SBL_ERR_DEVICE; ++s) {
        const char *t = sbl_status_string((sbl_status)s);
        CHECK(t != NULL && t[0] != '\0');
    }

    /* row bytes of every packed buffer, for a 6:8 and a 2:4 layer */
    const sbl_layer_desc d68 = {528, 1040, 6, 8};
    const sbl_layer_desc d24 = {96, 2560, 2, 4};
    CHECK(sbl_packed_row_bytes(&d68, SBL_FMT_PK2, SBL_BUF_MAIN) == round16(1040 / 4));
    CHECK(sbl_packed_row_bytes(&d68, SBL_FMT_NM, SBL_BUF_MAIN) == round16((1040 / 8 * 6 + 3) / 4));
    CHECK(sbl_packed_row_bytes(&d68, SBL_FMT_NM, SBL_BUF_NM_BITMAP) == round16(1040 / 8));
    CHECK(sbl_packed_row_bytes(&d68, SBL_FMT_I8, SBL_BUF_MAIN) == 1040);
    CHECK(sbl_packed_row_bytes(&d68, SBL_FMT_BF16T, SBL_BUF_MAIN) == 2 * 528);
    CHECK(sbl_packed_row_bytes(&d24, SBL_FMT_SP24, SBL_BUF_MAIN) == round16(2560 / 2));
    CHECK(sbl_packed_row_bytes(&d24, SBL_FMT_SP24, SBL_BUF_SP24_META) == round16(2560 / 8));
    CHECK(sbl_packed_row_bytes(&d24, SBL_FMT_T24, SBL_BUF_MAIN) == round16(2560 / 8));
    CHECK(sbl_packed_row_bytes(&d24, SBL_FMT_T24, SBL_BUF_T24_HI) == round16(2560 / 16));

    /* invalid descriptors give 0 bytes */
    const sbl_layer_desc bad_m = {128, 256, 3, 6};
    const sbl_layer_desc bad_k = {128, 250, 2, 4};
    const sbl_layer_desc bad_o = {100, 256, 2, 4};
    const sbl_layer_desc bad_n = {128, 256, 0, 4};
    CHECK(sbl_packed_row_bytes(&bad_m, SBL_FMT_I8, SBL_BUF_MAIN) == 0);
    CHECK(sbl_packed_row_bytes(&bad_k, SBL_FMT_I8, SBL_BUF_MAIN) == 0);
    CHECK(sbl_packed_row_bytes(&bad_o, SBL_FMT_I8, SBL_BUF_MAIN) == 0);
    CHECK(sbl_packed_row_bytes(&bad_n, SBL_FMT_I8, SBL_BUF_MAIN) == 0);
    CHECK(sbl_packed_row_bytes(NULL, SBL_FMT_I8, SBL_BUF_MAIN) == 0);
    CHECK(sbl_workspace_bytes(&bad_m, 0, SBL_OP_QUANTIZE_MASK_PACK) == 0);

    /* workspaces: a fixed packing workspace; the backward's grows with T */
    const size_t ws_pack = sbl_workspace_bytes(&d68, 0, SBL_OP_QUANTIZE_MASK_PACK);
    CHECK(ws_pack > 0 && ws_pack % 256 == 0);
    CHECK(sbl_workspace_bytes(&d68, 64, SBL_OP_BACKWARD) > 0);
    CHECK(sbl_workspace_bytes(&d68, 4096, SBL_OP_BACKWARD) > sbl_workspace_bytes(&d68, 64, SBL_OP_BACKWARD));
    CHECK(sbl_workspace_bytes(&d68, -1, SBL_OP_BACKWARD) == 0);

    /* the forward-format rule (host only): the sparse kernel for 2:4-fitting
     * masks with K >= 1024 and at least 8192 * 1024 outputs, else int8 */
    const sbl_layer_desc down = {1536, 8960, 2, 4};
    const sbl_layer_desc gate = {4864, 896, 2, 4};
    const sbl_layer_desc down68 = {1536, 8960, 6, 8};
    CHECK(sbl_forward_format(&down, 8192) == SBL_FMT_SP24);
    CHECK(sbl_forward_format(&down, 16) == SBL_FMT_I8);
    CHECK(sbl_forward_format(&gate, 4096) == SBL_FMT_I8);
    CHECK(sbl_forward_format(&down68, 8192) == SBL_FMT_I8);
    CHECK(sbl_forward_format(&bad_m, 8192) == 0);
    CHECK(sbl_forward_format(&down, -1) == 0);

    /* argument checks, all before any device access */
    sbl_packed w;
    memset(&w, 0, sizeof(w));
    w.i8 = (int8_t *)A;
    w.bf16t = (uint16_t *)A;
    w.gamma = (float *)B;
    CHECK(sbl_quantize_act(A, 4, 250, B, B, NULL) == SBL_ERR_SHAPE);
    CHECK(sbl_quantize_act(NULL, 4, 256, B, B, NULL) == SBL_ERR_INVALID_ARG);
    CHECK(sbl_quantize_act(MIS, 4, 256, B, B, NULL) == SBL_ERR_ALIGNMENT);
    CHECK(sbl_quantize_act(A, 0, 256, B, B, NULL) == SBL_OK);  /* no tokens: nothing to do */
    CHECK(sbl_quantize_act_rmsnorm(A, 4, 256, NULL, -1.0f, B, B, NULL) == SBL_ERR_INVALID_ARG);
    CHECK(sbl_forward(&bad_m, A, B, 4, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_ERR_UNSUPPORTED);
    CHECK(sbl_forward(&d68, A, B, -1, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_ERR_SHAPE);
    CHECK(sbl_forward(&d68, A, B, 0, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_OK);
    CHECK(sbl_forward(&d68, NULL, B, 4, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_ERR_INVALID_ARG);
    CHECK(sbl_forward(&d68, MIS, B, 4, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_ERR_ALIGNMENT);
    {
        /* the format's own buffers are checked once the device is known */
        const sbl_status st = sbl_forward(&d68, A, B, 4, &w, SBL_FMT_SP24, B, 0, NULL, NULL);
        CHECK(st == SBL_ERR_INVALID_ARG || (no_device && st == SBL_ERR_DEVICE));
    }
    CHECK(sbl_quantize_mask_pack(&d68, (const float *)A, SBL_FMT_I8, &w, NULL, 0, NULL) == SBL_ERR_WORKSPACE);
    CHECK(sbl_quantize_mask_pack(&d68, (const float *)A, 1u << 7, &w, B, 1 << 20, NULL) == SBL_ERR_INVALID_ARG);
    CHECK(sbl_quantize_mask_pack(&d68, (const float *)A, SBL_FMT_BF16T, &w, B, 1 << 20, NULL) ==
          SBL_ERR_UNSUPPORTED);
    CHECK(sbl_backward_dual_ste(&d68, A, NULL, NULL, 4, &w, NULL, 1, NULL, NULL, 0, NULL) ==
          SBL_ERR_INVALID_ARG);  /* neither dX nor dW asked for */
    CHECK(sbl_backward_dual_ste(&d68, A, A, B, 4, &w, NULL, 1, (float *)B, NULL, 0, NULL) ==
          SBL_ERR_WORKSPACE);
    CHECK(sbl_device_error(NULL, 0) == SBL_ERR_INVALID_ARG);

    /* the packed-layer container, host memory only */
    {
        static uint8_t pk2[16 * 16], i8[16 * 64], image[4096], back_pk2[16 * 16], back_i8[16 * 64];
        const sbl_layer_desc dc = {16, 64, 2, 4};
        for (size_t i = 0; i < sizeof(pk2); ++i) pk2[i] = (uint8_t)(i * 7 + 1);
        for (size_t i = 0; i < sizeof(i8); ++i) i8[i] = (uint8_t)(i % 3);
        sbl_host_buffers src, dst;
        memset(&src, 0, sizeof(src));
        memset(&dst, 0, sizeof(dst));
        src.pk2 = pk2;
        src.i8 = i8;
        dst.pk2 = back_pk2;
        dst.i8 = back_i8;
        const uint32_t fm = SBL_FMT_PK2 | SBL_FMT_I8;
        const size_t nb = sbl_container_bytes(&dc, fm);
        CHECK(nb == SBL_CONTAINER_HEADER_BYTES + sizeof(pk2) + sizeof(i8));
        CHECK(sbl_container_write(&dc, fm, 0.25f, &src, image, nb - 1) == SBL_ERR_SHAPE);
        CHECK(sbl_container_write(&dc, fm, 0.25f, &src, image, sizeof(image)) == SBL_OK);
        sbl_layer_desc di;
        uint32_t fi = 0;
        float gi = 0.0f;
        CHECK(sbl_container_info(image, nb, &di, &fi, &gi) == SBL_OK);
        CHECK(di.out_features == 16 && di.in_features == 64 && di.n == 2 && di.m == 4 && fi == fm && gi == 0.25f);
        CHECK(sbl_container_read(image, nb, &dst) == SBL_OK);
        CHECK(memcmp(back_pk2, pk2, sizeof(pk2)) == 0 && memcmp(back_i8, i8, sizeof(i8)) == 0);
        image[nb - 1] ^= 1u;
        CHECK(sbl_container_info(image, nb, NULL, NULL, NULL) == SBL_ERR_INVALID_ARG);
        CHECK(sbl_container_info(image, 10, NULL, NULL, NULL) == SBL_ERR_INVALID_ARG);
    }

    if (no_device) {
        /* valid calls: the only thing left is the device, which is absent */
        CHECK(sbl_quantize_act(A, 4, 256, B, B, NULL) == SBL_ERR_DEVICE);
        CHECK(sbl_forward(&d68, A, B, 4, &w, SBL_FMT_I8, B, 0, NULL, NULL) == SBL_ERR_DEVICE);
        CHECK(sbl_quantize_mask_pack(&d68, (const float *)A, SBL_FMT_I8, &w, B, ws_pack, NULL) == SBL_ERR_DEVICE);
        CHECK(sbl_selftest_wait_expiry(NULL) == SBL_ERR_DEVICE);
    }

    if (failures) {
        fprintf(stderr, "%d check(s) failed\n", failures);
        return 1;
    }
    printf("abi_host_check: all checks passed%s\n", no_device ? " (no device)" : "");
    return 0;
}
