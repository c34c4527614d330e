/* A plain C program against include/qift.h and libqift.so: the boundary needs no C++, no CUDA
 * headers and no torch.  Every call below is rejected (or is a no-op) during host-side
 * validation, so the program runs on a machine without a GPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "qift.h"

static int failures = 0;

static void expect(const char* what, qift_status got, qift_status want) {
    if (got != want) {
        printf("FAIL %s: %s, expected %s\n", what, qift_status_string(got), qift_status_string(want));
        ++failures;
    }
}

int main(void) {
    void* const fake = (void*)(uintptr_t)0x10000; /* 16-byte aligned, never dereferenced */
    void* const mis = (void*)(uintptr_t)0x10004;  /* misaligned */

    if (strcmp(qift_status_string(QIFT_OK), "QIFT_OK") != 0) {
        printf("FAIL status string of QIFT_OK: %s\n", qift_status_string(QIFT_OK));
        ++failures;
    }
    if (strncmp(qift_status_string(QIFT_ERR_TIMEOUT), "QIFT_ERR_TIMEOUT", 16) != 0) {
        printf("FAIL status string of QIFT_ERR_TIMEOUT: %s\n", qift_status_string(QIFT_ERR_TIMEOUT));
        ++failures;
    }

    expect("rotate: block not a power of two", qift_rotate(fake, fake, QIFT_F32, 4, 96, 3, NULL), QIFT_ERR_INVALID_ARG);
    expect("rotate: misaligned", qift_rotate(mis, fake, QIFT_F32, 4, 64, 64, NULL), QIFT_ERR_INVALID_ARG);
    expect("rotate: no rows", qift_rotate(NULL, NULL, QIFT_F16, 0, 64, 64, NULL), QIFT_OK);

    expect("quantize_weights: n_in % 16",
           qift_quantize_weights(fake, 4, 40, QIFT_SET_QIFT, 100, 0.2, 1.0, fake, fake, NULL, NULL),
           QIFT_ERR_INVALID_ARG);
    expect("quantize_weights: grid",
           qift_quantize_weights(fake, 4, 64, QIFT_SET_POT, 1, 0.2, 1.0, fake, fake, NULL, NULL),
           QIFT_ERR_INVALID_ARG);
    expect("quantize_weights: no rows",
           qift_quantize_weights(NULL, 0, 64, QIFT_SET_INT4, 100, 0.2, 1.0, NULL, NULL, NULL, NULL), QIFT_OK);

    expect("quantize_acts: block", qift_quantize_acts(fake, 2, 64, 3, fake, fake, NULL), QIFT_ERR_INVALID_ARG);
    expect("quantize_acts: no tokens", qift_quantize_acts(NULL, 0, 64, 0, NULL, NULL, NULL), QIFT_OK);

    expect("linear: standard set", qift_linear(fake, fake, fake, fake, QIFT_SET_STD, 1, 8, 64, fake, QIFT_F16, NULL),
           QIFT_ERR_UNSUPPORTED);
    expect("linear: 17 tokens, n_in not a multiple of 64",
           qift_linear(fake, fake, fake, fake, QIFT_SET_QIFT, 17, 8, 80, fake, QIFT_F16, NULL), QIFT_ERR_UNSUPPORTED);
    expect("linear: 4-bit, n_in not a multiple of 64",
           qift_linear(fake, fake, fake, fake, QIFT_SET_INT4, 17, 8, 48, fake, QIFT_F16, NULL), QIFT_ERR_UNSUPPORTED);
    expect("linear: no tokens", qift_linear(NULL, NULL, NULL, NULL, QIFT_SET_QIFT, 0, 8, 64, NULL, QIFT_F32, NULL),
           QIFT_OK);

    expect("decode_linear: five tokens",
           qift_decode_linear(fake, 5, 128, 128, fake, fake, QIFT_SET_INT4, 8, fake, QIFT_F16, NULL, NULL, NULL),
           QIFT_ERR_UNSUPPORTED);
    expect("decode_linear: standard set",
           qift_decode_linear(fake, 1, 128, 128, fake, fake, QIFT_SET_STD, 8, fake, QIFT_F16, NULL, NULL, NULL),
           QIFT_ERR_UNSUPPORTED);
    expect("quantize_kv: block", qift_quantize_kv(fake, 2, 64, 3, fake, fake, NULL), QIFT_ERR_INVALID_ARG);
    expect("dequantize_kv: no tokens", qift_dequantize_kv(NULL, NULL, 0, 64, 64, NULL, NULL), QIFT_OK);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
