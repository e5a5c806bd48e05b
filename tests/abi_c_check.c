/* A plain C11 client of the library: the header compiles as C, the library links
 * and loads, and host-side argument checks answer without a GPU.  Exit status 0 on
 * success; each failed check prints its line. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ep_b200.h"

static int failures = 0;
#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                          \
        }                                                        \
    } while (0)

int main(void) {
    CHECK(ep_abi_version() == 2);
    CHECK(strcmp(ep_status_string(EP_ERR_SHAPE), "unsupported size") == 0);
    CHECK(ep_workspace_bytes(4096, 256, 8) > 0);
    CHECK(ep_workspace_bytes(-1, 256, 8) == 0);

    /* shape and pointer checks run before anything touches CUDA */
    uintptr_t fake = 0x100000;
    void* f = (void*)fake;
    ep_layout lay;
    lay.num_tokens_per_expert = lay.num_tokens_per_partition = lay.expert_offset = lay.row_of =
        lay.src_of = lay.num_recv = (int32_t*)f;
    lay.is_token_in_partition = (uint8_t*)f;
    CHECK(ep_get_dispatch_layout(4, 0, 8, 2, (const int64_t*)f, &lay, f, 1u << 20, NULL) ==
          EP_ERR_SHAPE);
    CHECK(ep_dispatch(16, 256, 4, 8, 2, EP_QUANT_FP8_E4M3_1X128 | EP_QUANT_SCALES_MN_MAJOR, f,
                      (const int64_t*)f, (const float*)f, f, NULL, (int32_t*)f, (float*)f, &lay,
                      f, 1u << 20, NULL) == EP_ERR_INVALID_ARG);
    CHECK(ep_combine(0, 128, 2, NULL, 0, &lay, NULL, NULL, f, 4096, NULL) == EP_OK);

    ep_peer_buffers peers;
    peers.recv_x = (void* const*)f;
    peers.recv_scales = (float* const*)f;
    peers.recv_topk_idx = (int32_t* const*)f;
    peers.recv_topk_weights = (float* const*)f;
    peers.capacity = (int64_t)1 << 31;
    CHECK(ep_peer_dispatch(16, 256, 4, 8, 2, EP_QUANT_FP8_E4M3_1X128, f, (const int64_t*)f,
                           (const float*)f, &lay, (const int32_t*)f, &peers, f, 4096, NULL) ==
          EP_ERR_SHAPE);
    CHECK(ep_peer_plan(3, 0, 8, (const int32_t*)f, (const int32_t*)f, 64, (int32_t*)f,
                       (int32_t*)f, (int32_t*)f, f, 4096, NULL) == EP_ERR_SHAPE);
    void* ptr = NULL;
    char handle[EP_IPC_HANDLE_BYTES];
    CHECK(ep_ipc_alloc(0, &ptr, handle) == EP_ERR_INVALID_ARG);
    CHECK(ep_ipc_close(NULL) == EP_ERR_INVALID_ARG);

    if (failures == 0) printf("ok\n");
    return failures == 0 ? 0 : 1;
}
