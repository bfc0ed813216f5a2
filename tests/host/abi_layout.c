/* Prints sizeof and field offsets of the C ABI's structs, so the Python binding's ctypes mirrors
 * can be checked against the header as the C compiler lays it out. */
#include <stddef.h>
#include <stdio.h>

#include "moe.h"

#define F(S, m) printf(#S " " #m " %zu %zu\n", offsetof(S, m), sizeof(((S*)0)->m))

int main(void) {
  printf("moe_config_t sizeof %zu\n", sizeof(moe_config_t));
  F(moe_config_t, T); F(moe_config_t, d); F(moe_config_t, E); F(moe_config_t, k);
  F(moe_config_t, d_ff); F(moe_config_t, n_shared); F(moe_config_t, act);
  F(moe_config_t, gate_norm); F(moe_config_t, capacity_factor); F(moe_config_t, capacity);
  F(moe_config_t, dtype); F(moe_config_t, has_bias); F(moe_config_t, aux_loss_coef);
  F(moe_config_t, drop_order);
  printf("moe_layout_t sizeof %zu\n", sizeof(moe_layout_t));
  F(moe_layout_t, capacity); F(moe_layout_t, T_pad); F(moe_layout_t, rows);
  F(moe_layout_t, routed_row0); F(moe_layout_t, max_group_rows); F(moe_layout_t, ctx_logits);
  F(moe_layout_t, ctx_topk_idx); F(moe_layout_t, ctx_topk_w); F(moe_layout_t, ctx_counts);
  F(moe_layout_t, ctx_kept); F(moe_layout_t, ctx_offsets); F(moe_layout_t, ctx_slot);
  F(moe_layout_t, ctx_row_token); F(moe_layout_t, ctx_Xd); F(moe_layout_t, ctx_Gu);
  F(moe_layout_t, ctx_Gv); F(moe_layout_t, ctx_H); F(moe_layout_t, ctx_O);
  F(moe_layout_t, ctx_bytes); F(moe_layout_t, scratch_bytes); F(moe_layout_t, ctx_aux_loss);
  return 0;
}
