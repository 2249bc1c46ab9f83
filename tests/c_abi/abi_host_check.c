/* A plain C99 client of include/bbc.h: it compiles the header as C, links libbbc.so and
 * exercises calls that the library rejects on the host (no GPU needed, nothing is launched),
 * plus the host-only normal-float codebook. Exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "bbc.h"

static int failures = 0;

static void expect(const char* what, int got, int want) {
    if (got != want) {
        printf("FAIL %s: status %d, expected %d (%s)\n", what, got, want, bbc_last_error());
        failures++;
    }
}

int main(void) {
    /* never dereferenced: every call below fails validation first */
    void* fake = (void*)(uintptr_t)0x100000;
    float cb4[16];

    expect("codebook K=4", bbc_nf_codebook(4, cb4), BBC_OK);
    if (cb4[15] != 1.0f || cb4[0] >= cb4[1]) {
        printf("FAIL codebook K=4 values\n");
        failures++;
    }
    expect("codebook K=9", bbc_nf_codebook(9, cb4), BBC_ERR_INVALID);

    expect("quantize null A", kbit_quantize(NULL, BBC_BF16, 64, 4, 32, fake, fake, fake, NULL), BBC_ERR_INVALID);
    expect("quantize K=6", kbit_quantize(fake, BBC_BF16, 64, 6, 32, fake, fake, fake, NULL), BBC_ERR_INVALID);
    expect("quantize bs=64", kbit_quantize(fake, BBC_BF16, 64, 4, 64, fake, fake, fake, NULL), BBC_ERR_UNSUPPORTED);
    expect("dequantize n=0", kbit_dequantize(fake, fake, fake, 4, 32, 0, BBC_F32, fake, NULL), BBC_ERR_INVALID);
    if (strlen(bbc_last_error()) == 0) {
        printf("FAIL no message for the last error\n");
        failures++;
    }
    expect("nested bs2=128",
           dequantize_4bit_nested(fake, fake, fake, fake, 0.0f, fake, 64, 64, 128, BBC_BF16, fake, NULL),
           BBC_ERR_UNSUPPORTED);
    expect("linear_kbit bits=6",
           linear_kbit(fake, BBC_BF16, 1, 16, 64, fake, fake, fake, 6, 32, fake, NULL), BBC_ERR_INVALID);
    expect("linear_4bit_nested M=33",
           linear_4bit_nested(fake, BBC_BF16, 33, 16, 64, fake, fake, fake, fake, 0.0f, fake, 64, 256, fake, NULL),
           BBC_ERR_UNSUPPORTED);
    expect("workspace bytes", (int)(quantize_4bit_nested_workspace_bytes(0, 64) == 0), 1);

    if (failures == 0) printf("c abi ok\n");
    return failures == 0 ? 0 : 1;
}
