/* A plain C client of libvc: includes only include/vc.h, links libvc.so, and calls the entry
 * points that need no device (sizes, host-side validation, status strings) for the tiny hybrid
 * model (d 256, pattern "M-*-", W8 g64).  Prints the sizes and "ok", or the failing check. */
#include <stdio.h>
#include <string.h>

#include "../../include/vc.h"

#define CHECK(c)                                   \
    do {                                           \
        if (!(c)) {                                \
            printf("failed: %s\n", #c);            \
            return 1;                              \
        }                                          \
    } while (0)

int main(void) {
    vc_config c;
    memset(&c, 0, sizeof(c));
    c.d_model = 256;
    c.pattern = "M-*-";
    c.ssm_heads = 8; c.ssm_head_dim = 32; c.ssm_state = 16; c.ssm_groups = 1;
    c.conv_width = 4; c.norm_groups = 1;
    c.attn_q_heads = 4; c.attn_kv_heads = 2; c.attn_head_dim = 64;
    c.mlp_hidden = 1024; c.vocab_text = 1024; c.vocab_func = 1024;
    c.eps = 1e-5f;
    c.wfmt = VC_W_INT8_SYM; c.group_size = 64; c.head_fmt = VC_W_INT8_SYM;
    c.max_batch = 1; c.kv_capacity = 128; c.n_slots = 1;

    size_t ws = vc_workspace_bytes(&c);
    size_t w_in = vc_weight_bytes(VC_W_INT8_SYM, 64, 8 * 32 * 2 + 2 * 16 + 8, 256);   /* in_proj */
    printf("workspace %zu\nin_proj %zu\n", ws, w_in);
    CHECK(ws > 0 && ws % 256 == 0);
    CHECK(w_in > 0);

    vc_config bad = c;
    bad.max_batch = 17;
    CHECK(vc_workspace_bytes(&bad) == 0);
    bad = c;
    bad.pattern = "M-x-";
    CHECK(vc_workspace_bytes(&bad) == 0);

    vc_backbone* h = (vc_backbone*)&c;   /* must be overwritten with NULL on failure */
    CHECK(vc_backbone_create(&c, NULL, NULL, ws, NULL, &h) == VC_ERR_INVALID_ARG);
    CHECK(h == NULL);
    CHECK(vc_step(NULL, NULL, 1, NULL, NULL, NULL, NULL, NULL) == VC_ERR_INVALID_ARG);
    CHECK(vc_prefill(NULL, NULL, 4, 0, NULL, NULL) == VC_ERR_INVALID_ARG);
    CHECK(strcmp(vc_status_string(VC_OK), "ok") == 0);
    vc_destroy(NULL);
    printf("ok\n");
    return 0;
}
