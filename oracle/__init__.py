"""Oracle for the SambaY scan + Gated Memory Unit hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It is a plain, slow,
obviously-correct CPU restatement of what the method computes, in float64,
written from the method's definition and sharing no code with the CUDA path.

Sources (cited per function in :mod:`oracle.sambay_ref`):

* "Decoder-Hybrid-Decoder Architecture for Efficient Reasoning with Long
  Generation", Paper-Notes page, section 方法详解 > 关键设计 (Gated Memory
  Unit): the GMU equation ``Y = (M ⊙ SiLU(X W1^T)) W2``, sigma = SiLU, the
  lifted mixing tensor ``Ã_ijk = G_ik A_ij`` and the constant-size decode
  state; section 方法详解 > 整体框架: prefill runs only the self-decoder,
  decode reuses the memory readout.
* The same paper's abstract (chatpaper.ai page, English abstract): the GMU
  shares "memory readout states" of the Samba self-decoder.
* Mamba selective SSM (Gu & Dao 2023, "Mamba: Linear-Time Sequence Modeling
  with Selective State Spaces", section 3.2 and its Algorithm 2 "SSM +
  Selection", section 3.4 architecture block): causal depthwise conv + SiLU,
  input-dependent Δ/B/C projections, softplus Δ, Ā = exp(ΔA), B̄ = ΔB,
  the recurrence and its readout.  Used as mathematics only.

* Mamba-2's SSD layer (Dao & Gu 2024, "Transformers are SSMs"), for the
  SambaY-2 ablation row (Paper-Notes page, 实验关键数据 > 消融实验): one
  scalar decay per head, B and C shared by the heads; in
  :mod:`oracle.ssd_ref`.  Used as mathematics only.

Parity status per function: every function is pinned by a CPU test in
``tests/test_oracle_pins.py`` against something other than itself (closed
forms, brute force, library routines, hand-derived golden values).  The one
thing no test can pin is agreement with the paper's trained model (there are
no printed activations or weights); that is "parity unpinned" and stated so.
"""

from .sambay_ref import (  # noqa: F401
    silu,
    softplus,
    causal_conv1d_silu,
    x_proj,
    dt_softplus,
    selective_scan,
    scan_prefill_ref,
    scan_step_ref,
    gmu_ref,
    gmu_layers_ref,
    mixing_matrix_ref,
    lifted_gmu_ref,
    round_bf16,
    mamba_layer_ref,
    mlp_representation_ref,
    sambay_mlp_gmu_ref,
    cross_attention_decode_ref,
)
from .ssd_ref import (  # noqa: F401
    ssd_recurrent,
    ssd_chunked,
    ssd_matrix,
    mamba2_scan_ref,
    mamba2_step_ref,
)
