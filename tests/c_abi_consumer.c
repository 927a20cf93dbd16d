/*
 * A C99 program that uses the library only through include/deltalog.h: it prints
 * the struct layouts it sees (so that the test can compare them with the Python
 * binding's) and makes the calls that need no GPU.  Built and run by
 * tests/test_abi.py.
 */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "deltalog.h"

#define FIELD(T, f) printf("%s.%s %zu\n", #T, #f, offsetof(T, f))

static int fails = 0;
static void expect(int cond, const char *what) {
    if (!cond) {
        printf("FAIL %s\n", what);
        fails++;
    }
}

int main(void) {
    printf("sizeof.dl_pool_desc %zu\n", sizeof(dl_pool_desc));
    printf("sizeof.dl_step_args %zu\n", sizeof(dl_step_args));
    FIELD(dl_pool_desc, n_slots);
    FIELD(dl_pool_desc, log_cap);
    FIELD(dl_pool_desc, decay);
    FIELD(dl_pool_desc, update);
    FIELD(dl_pool_desc, tile_v);
    FIELD(dl_pool_desc, log_format);
    FIELD(dl_pool_desc, replay_mode);
    FIELD(dl_pool_desc, state);
    FIELD(dl_pool_desc, log);
    FIELD(dl_pool_desc, log_len);
    FIELD(dl_pool_desc, arrive);
    FIELD(dl_pool_desc, err_word);
    FIELD(dl_step_args, slots);
    FIELD(dl_step_args, batch);
    FIELD(dl_step_args, q);
    FIELD(dl_step_args, k);
    FIELD(dl_step_args, v);
    FIELD(dl_step_args, in_dtype);
    FIELD(dl_step_args, lambda);
    FIELD(dl_step_args, lambda_per_head);
    FIELD(dl_step_args, beta);
    FIELD(dl_step_args, out);

    /* a descriptor naming aligned placeholder addresses: nothing is dereferenced
       on the host, and no call below reaches the device */
    dl_pool_desc d;
    memset(&d, 0, sizeof d);
    d.n_slots = 4;
    d.n_layers = 2;
    d.n_heads = 4;
    d.n_kheads = 2;
    d.d_k = 128;
    d.d_v = 128;
    d.log_cap = 8;
    d.decay = DL_DECAY_DIAG;
    d.update = DL_UPDATE_DELTA;
    d.tile_v = 0;
    d.log_format = DL_LOG_FP32;
    d.replay_mode = DL_REPLAY_PER_TILE;
    d.state = (float *)(uintptr_t)0x10000;
    d.log = (float *)(uintptr_t)0x20000;
    d.log_len = (int32_t *)(uintptr_t)0x30000;
    d.arrive = (int32_t *)(uintptr_t)0x40000;
    d.err_word = (int32_t *)(uintptr_t)0x50000;

    int64_t bytes = 0;
    expect(dl_log_bytes(&d, &bytes) == DL_OK, "dl_log_bytes");
    /* 4 slots x 2 layers x 4 heads x 8 entries x (128 + 128 + 128) floats */
    expect(bytes == (int64_t)4 * 2 * 4 * 8 * 384 * 4, "fp32 log bytes");
    printf("log_bytes %lld\n", (long long)bytes);

    dl_pool *pool = NULL;
    expect(dl_create_pool(&d, &pool) == DL_OK && pool != NULL, "dl_create_pool");
    dl_step_args a;
    memset(&a, 0, sizeof a);
    a.slots = (const int32_t *)(uintptr_t)0x60000;
    a.batch = 0; /* an empty batch is valid and launches nothing */
    a.q = a.k = a.v = (const void *)(uintptr_t)0x60000;
    a.in_dtype = DL_BF16;
    a.lambda = (const float *)(uintptr_t)0x60000;
    a.beta = (const float *)(uintptr_t)0x60000;
    a.out = (float *)(uintptr_t)0x60000;
    expect(dl_decode_step(pool, 0, &a, 1, NULL) == DL_OK, "empty decode step");
    a.batch = 5; /* more rows than slots */
    expect(dl_decode_step(pool, 0, &a, 1, NULL) == DL_ERR_SHAPE, "oversized batch");
    expect(dl_read_error(pool, NULL, 0, NULL) == DL_ERR_INVALID_ARG, "read_error without output");
    expect(dl_destroy_pool(pool) == DL_OK, "dl_destroy_pool");

    /* the allocation-free step: host checks only (batch 0 returns before any CUDA call) */
    a.batch = 0;
    expect(dl_decode_step_noalloc(&d, 0, &a, DL_MERGE_ADAPTIVE, NULL) == DL_OK, "noalloc empty step");
    expect(dl_decode_step_noalloc(NULL, 0, &a, DL_MERGE_ADAPTIVE, NULL) == DL_ERR_INVALID_ARG,
           "noalloc without descriptor");
    expect(dl_decode_step_noalloc(&d, 2, &a, DL_MERGE_ADAPTIVE, NULL) == DL_ERR_INVALID_ARG,
           "noalloc layer out of range");
    {
        dl_pool_desc big = d;
        big.n_slots = DL_NOALLOC_MAX_COUNTERS; /* x 2 layers: more counters than the array */
        expect(dl_decode_step_noalloc(&big, 0, &a, DL_MERGE_ADAPTIVE, NULL) == DL_ERR_SHAPE,
               "noalloc counter limit");
    }

    /* merge policy: at capacity never merges every step; adaptive does below a few
       heads per SM (one 32-head slot) and does not for a launch that fills the GPU */
    int32_t every = -1;
    expect(dl_merge_policy(1, 32, DL_MERGE_ADAPTIVE, NULL) == DL_ERR_INVALID_ARG, "merge_policy without output");
    expect(dl_merge_policy(-1, 32, DL_MERGE_ADAPTIVE, &every) == DL_ERR_INVALID_ARG, "merge_policy negative batch");
    expect(dl_merge_policy(1, 32, DL_MERGE_AT_CAPACITY, &every) == DL_OK && every == 0, "capacity policy");
    expect(dl_merge_policy(1, 32, DL_MERGE_ADAPTIVE, &every) == DL_OK && every == 1, "adaptive, one slot");
    expect(dl_merge_policy(256, 32, DL_MERGE_ADAPTIVE, &every) == DL_OK && every == 0, "adaptive, full launch");
    printf("merge_policy ok\n");

    /* the stall test hook is host state only; 0 switches it off */
    expect(dl_debug_stall(0) == DL_OK, "dl_debug_stall off");
    expect(dl_status_string(DL_OK) != NULL && dl_status_string(DL_ERR_SHAPE) != NULL, "status strings");

    d.d_k = 0;
    expect(dl_create_pool(&d, &pool) == DL_ERR_SHAPE, "bad d_k refused");
    printf("%s\n", fails ? "FAILED" : "OK");
    return fails ? 1 : 0;
}
