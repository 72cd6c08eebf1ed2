"""CPU oracle for the Dust per-token activation-space gradient estimator.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, fp64 NumPy
restatement of what the estimator computes. Only the tests, the smoke check
of ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it;
the library's product path never does, and it shares no code with the CUDA
path (only the seeded input generators in ``synth`` serve both).

Sources (the Dust pages, cited by title and section):

* "Dust：无需反向传播的Transformer零阶预训练" (agentlenshq), §1
  "Dust的不同之处": per-token Gaussian noise on each linear layer's output
  (激活空间扰动); reward = loss reduction at the token, estimate
  g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i), weight gradient
  G_W = sum_t g_t x_t^T (无需反向传播的信用分配); the LM head is perturbed on
  cached logits with a small vocabulary subset per draw, layer types in
  separate passes (减少干扰). §2 "实证发现", 梯度对齐: cos(K) law.
* "不用反向传播训练Transformer：Dust零阶优化获突破" (tahou): the paragraph on
  interference reductions (separate passes per layer type, cached unperturbed
  intermediates, LM head on cached logits recomputing only the loss).
* "Dust: предобучение трансформеров без обратного распространения ошибки"
  (iitog), "Механика такая": noise on each linear layer's output, independent
  per token; reward-weighted noise average is the output-error estimate, its
  outer product with the layer input the weight gradient.
* The attention-internals variant (``attn.py``) follows §1 of the first page
  (the attention internals' reward comes from the change of the attention
  output; only the attention output is recomputed per draw) and the second
  page's remark that this change is judged together with an error signal.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against closed forms, invariants, brute-force finite differences, library
routines and published known-answer vectors. No function is unpinned.
"""
from .philox import (  # noqa: F401
    philox4x32_10,
    box_muller,
    slot_counter_word,
    gaussians,
    subset_offset,
    default_subset_a,
    TAG_HEAD,
    TAG_SUBSET_OFFSET,
    TAG_MLP_UP,
    TAG_MLP_DOWN,
    TAG_ATTN_OUT,
    TAG_ATTN_Q,
    TAG_ATTN_K,
    TAG_ATTN_V,
)
from .params import Params  # noqa: F401
from .head import (  # noqa: F401
    clean_head, head_grad, head_linear_estimate, full_vocab_draws, subset_draws,
)
from .mlp import (  # noqa: F401
    clean_mlp, mlp_grad, mlp_draws, gelu, mlp_down_grad, mlp_down_draws, attn_out_grad,
    attn_out_draws,
)
from .optim import sgd_momentum, train_head, exact_weight_grad  # noqa: F401
from .attn import attention, attention_seq, attn_draws, attn_grad, perturbed_outputs  # noqa: F401
