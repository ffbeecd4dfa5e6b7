"""Plain, slow CPU fp64 oracle for the forward pass of one DECO MoE FFN layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline /
reference arm may import or run it.  It shares no code with the CUDA library
(`sparse_moe_ffn_relu_b200`); the only module both sides use is `synth`, the
seeded input generator, which holds none of the layer's arithmetic.

Sources, cited by page title and section:

[arXiv]  "DECO: Sparse Mixture-of-Experts with Dense-Comparable Performance on
         End-Side Devices" (arXiv 2605.10933, HTML edition): §1 Introduction;
         §2 Related work, paragraphs "Router design" and "Expert design";
         §5 acceleration-kernel experiment.
[press]  the qidianchuan.cn press summary of the same paper, part 2 ("DECO的
         核心设计", the core design): the router paragraph (ReLU routing,
         expert-wise scaling, shared expert) and the expert-design paragraphs
         (NormSiLU's two normalisation steps, precomputed mean, non-gated MLP
         experts).

What the layer computes (one token x_t, fp64 throughout, operands as stored):

1. Router logits z_e = b_r[e] + sum_k x_t[k] W_r[e,k]; expert e is active iff
   z_e > 0 (a zero or negative score is ignored), r_e = ReLU(z_e) is used raw
   -- no softmax / sigmoid / unit-sum renormalisation ([press] router
   paragraph; [arXiv] §1 and §2 "Router design").
2. Mean up-projection u = W_bar_up x_t, W_bar_up = (1/E) sum_e W_up[e], fixed
   at inference ([press] NormSiLU paragraph and the precompute remark).
3. For each active e (ascending): g = W_up[e] x_t; c = g - u (inter-expert
   mean normalisation); h = c / sqrt(mean_j c_j^2 + eps) (intra-expert RMS
   normalisation, no gain); a = SiLU(h) = h / (1 + exp(-h)); v_e = W_down[e] a
   ([press] NormSiLU paragraph; [arXiv] §1 "dual-stage normalization prior to
   the SiLU operator"; non-gated experts: [press] and [arXiv] §2 "Expert
   design").
4. Shared expert S = W_s_down SiLU(W_s_up x_t) (always on; [press] router
   paragraph, [arXiv] §1).
5. y_t = S + sum_{e active, ascending} s_e r_e v_e ([press] expert-wise router
   scaling; [arXiv] §1 "learnable expert-wise router scaling").

Readings where the pages are silent (shared with the CUDA path, each listed
in the design notes): strict z > 0; bias b_r present; eps = 1e-6 inside the
square root; no RMS gain; the mean runs over all E routed experts only; the
shared expert uses plain SiLU; y is rounded once to the storage dtype.

Exact routing decision: every product x_k * W_r[e,k] of two bf16 or two fp32
values is exact in fp64 (at most 16 or 48 significant bits), and
`math.fsum` returns the correctly rounded sum of its arguments, whose sign is
the sign of the exact real sum.  So the oracle's active set is the exact one.

Parity pins: see tests/test_oracle.py.  Parity unpinned (documented choices
that the pages do not fix): the value of eps, the absence of a gain, the
shared expert's activation and the router bias.
"""
from .deco import (  # noqa: F401
    to_f64, round_bf16, round_storage, silu, router_logits, route, routing_tables,
    mean_up, norm_silu, expert_output, shared_expert, layer_forward,
    layer_forward_tokens, dense_ffn, stack_forward, topk_route, exact_logit,
)
from .backward import (  # noqa: F401
    silu_grad, norm_silu_backward, layer_backward_tokens, router_entropy, sparsity_controller,
)
