/* Prints the size of every struct include/vc.h declares and the offset of each member, as
 * "struct.member offset" lines and "struct size" lines, compiled as plain C (C99) with the host
 * compiler.  The Python binding's ctypes structures must agree with these numbers. */
#include <stddef.h>
#include <stdio.h>

#include "../../include/vc.h"

#define SZ(T) printf("%s %zu\n", #T, sizeof(T))
#define OFF(T, m) printf("%s.%s %zu\n", #T, #m, offsetof(T, m))

int main(void) {
    SZ(vc_config);
    OFF(vc_config, d_model); OFF(vc_config, pattern); OFF(vc_config, ssm_heads); OFF(vc_config, ssm_head_dim);
    OFF(vc_config, ssm_state); OFF(vc_config, ssm_groups); OFF(vc_config, conv_width); OFF(vc_config, norm_groups);
    OFF(vc_config, attn_q_heads); OFF(vc_config, attn_kv_heads); OFF(vc_config, attn_head_dim);
    OFF(vc_config, mlp_hidden); OFF(vc_config, vocab_text); OFF(vc_config, vocab_func); OFF(vc_config, eps);
    OFF(vc_config, wfmt); OFF(vc_config, group_size); OFF(vc_config, head_fmt); OFF(vc_config, max_batch);
    OFF(vc_config, kv_capacity); OFF(vc_config, n_slots);
    SZ(vc_qmat);
    OFF(vc_qmat, data); OFF(vc_qmat, fmt); OFF(vc_qmat, group); OFF(vc_qmat, N); OFF(vc_qmat, K);
    SZ(vc_layer_weights);
    OFF(vc_layer_weights, norm); OFF(vc_layer_weights, in_proj); OFF(vc_layer_weights, out_proj);
    OFF(vc_layer_weights, conv_w); OFF(vc_layer_weights, conv_b); OFF(vc_layer_weights, A_log);
    OFF(vc_layer_weights, D); OFF(vc_layer_weights, dt_bias); OFF(vc_layer_weights, gnorm);
    OFF(vc_layer_weights, qkv); OFF(vc_layer_weights, o); OFF(vc_layer_weights, up); OFF(vc_layer_weights, down);
    SZ(vc_weights);
    OFF(vc_weights, layers); OFF(vc_weights, final_norm); OFF(vc_weights, head_text); OFF(vc_weights, head_func);
    SZ(vc_state);
    OFF(vc_state, ssm); OFF(vc_state, conv); OFF(vc_state, k); OFF(vc_state, v); OFF(vc_state, ctx_len);
    OFF(vc_state, status);
    SZ(vc_token_embeddings);
    OFF(vc_token_embeddings, emb_text); OFF(vc_token_embeddings, emb_func);
    return 0;
}
