/*
 * abi_consumer.c -- a plain C99 consumer of the libmpt C ABI (include/mpt.h).
 *
 * Built and run by tests/test_abi.py with gcc -std=c99 -Wall -Wextra
 * -Wpedantic -Werror and linked against libmpt.so.  It takes the address of
 * every entry point the header declares (so linking fails if the library
 * lacks one) and calls only what needs no GPU: configuration defaults,
 * workspace sizing, shard lengths, error strings and the argument errors of
 * every call on a NULL handle.  Exit status 0 = every check held.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mpt.h"

#define CHECK(cond)                                                             \
    do {                                                                        \
        if (!(cond)) {                                                          \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond);  \
            return 1;                                                           \
        }                                                                       \
    } while (0)

typedef void (*entry_fn)(void);

int main(void)
{
    /* every declared entry point, resolved by the linker */
    const entry_fn entries[] = {
        (entry_fn)mpt_config_init,       (entry_fn)mpt_workspace_bytes,
        (entry_fn)mpt_create,            (entry_fn)mpt_tensor_views,
        (entry_fn)mpt_refresh_half,      (entry_fn)mpt_step,
        (entry_fn)mpt_step_async,        (entry_fn)mpt_wait,
        (entry_fn)mpt_device_scale,      (entry_fn)mpt_shard_len,
        (entry_fn)mpt_step_partial,      (entry_fn)mpt_step_finish,
        (entry_fn)mpt_grad_histogram,    (entry_fn)mpt_stats,
        (entry_fn)mpt_get_scaler_state,  (entry_fn)mpt_set_scaler_state,
        (entry_fn)mpt_set_timing,        (entry_fn)mpt_debug_fail_next_step,
        (entry_fn)mpt_destroy,           (entry_fn)mpt_error_string,
        (entry_fn)mpt_check_flat_noalloc,
    };
    for (size_t i = 0; i < sizeof entries / sizeof entries[0]; ++i)
        CHECK(entries[i] != NULL);

    /* configuration defaults */
    mpt_config c;
    memset(&c, 0xFF, sizeof c);
    CHECK(mpt_config_init(&c) == MPT_OK);
    CHECK(c.backoff == 0.5f && c.growth == 2.0f);
    CHECK(c.flags == 0 && c.check_chunk_elems == 0 && c.update_chunk_elems == 0);
    CHECK(c.scaler_mode == MPT_SCALER_DYNAMIC && c.optimizer == MPT_OPT_MOMENTUM);
    CHECK(c.direct_margin == 2.0f && c.min_scale > 0.0f && c.max_scale >= c.min_scale);
    CHECK(mpt_config_init(NULL) == MPT_ERR_INVALID_ARG);

    /* workspace sizing: three arenas (4 + 4 + 2 bytes per element) plus tables */
    const int64_t one[1] = {1000000};
    size_t bytes = 0;
    CHECK(mpt_workspace_bytes(one, 1, NULL, &bytes) == MPT_OK);
    CHECK(bytes >= (size_t)10 * 1000000 && bytes < (size_t)10 * 1000000 + 65536);
    const int64_t bad[2] = {5, 0};
    CHECK(mpt_workspace_bytes(bad, 2, NULL, &bytes) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_workspace_bytes(NULL, 1, NULL, &bytes) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_workspace_bytes(one, 1, &c, NULL) == MPT_ERR_INVALID_ARG);

    /* shard lengths: equal shards, rounded up to 16 elements */
    int64_t n = 0;
    CHECK(mpt_shard_len(100003, 2, &n) == MPT_OK && n == 50016);
    CHECK(mpt_shard_len(0, 2, &n) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_shard_len(10, 0, &n) == MPT_ERR_INVALID_ARG);

    /* every status has a message */
    for (int code = 1; code >= -7; --code) {
        const char* s = mpt_error_string(code);
        CHECK(s != NULL && s[0] != '\0');
    }

    /* NULL handles are argument errors, and nothing is touched */
    mpt_step_result r;
    mpt_stats_t st;
    float f = 0.0f;
    int32_t k = 0;
    float* fp = NULL;
    void* vp = NULL;
    uint64_t hist[32];
    const void* ptrs[1] = {NULL};
    CHECK(mpt_step(NULL, ptrs, 1.0f, 0.1f, 0.9f, 0.0f, 0.0f, NULL, &r) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_step_async(NULL, ptrs, 0.1f, 0.9f, 0.0f, 0.0f, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_wait(NULL, NULL, &r) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_refresh_half(NULL, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_tensor_views(NULL, 0, &fp, &fp, &vp) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_device_scale(NULL, &fp) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_step_partial(NULL, ptrs, NULL, &vp) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_step_finish(NULL, NULL, 1, 0.1f, 0.9f, 0.0f, 0.0f, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_grad_histogram(NULL, hist) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_stats(NULL, &st) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_get_scaler_state(NULL, &f, &k) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_set_scaler_state(NULL, 1.0f, 0) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_set_timing(NULL, 1) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_debug_fail_next_step(NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_destroy(NULL) == MPT_OK);

    /* the allocation-free check rejects bad arguments before any CUDA call
       (the buffer addresses below are never dereferenced) */
    void* fake = (void*)(uintptr_t)0x10000;
    mpt_check_result* out = (mpt_check_result*)(uintptr_t)0x20000;
    CHECK(mpt_check_flat_noalloc(NULL, 10, 1.0f, 0.0f, out, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_check_flat_noalloc(fake, 0, 1.0f, 0.0f, out, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_check_flat_noalloc(fake, 10, 0.0f, 0.0f, out, NULL) == MPT_ERR_INVALID_ARG);
    CHECK(mpt_check_flat_noalloc(fake, MPT_NOALLOC_MAX_ELEMS + 1, 1.0f, 0.0f, out, NULL) ==
          MPT_ERR_TOO_LARGE);

    printf("abi consumer: %zu entry points, all checks passed\n",
           sizeof entries / sizeof entries[0]);
    return 0;
}
