"""CPU oracle for content-adaptive block-sparse tile attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use
it.  It is a plain, slow, fp64 restatement of the method, written so that a
reader can check it step by step against the source it cites.

Sources (cited by page title and section):

* "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science
  explanation of arXiv 2507.13546), section "Méthodologie : NABLA":
  token reordering ("Fractal Flattening"), block mean-pooling
  ("Sous-échantillonnage"), the reduced attention map ("Attention Réduite"),
  the per-row CDF threshold ("Seuil CDF"), expansion of the block mask
  ("Expansion") and the union with Sliding Tile Attention ("Intégration
  Hybride avec STA"); the lay section "L'ancienne solution" describes STA as
  a tile attending to itself and its direct neighbours.
* "AB-Attention accélère la génération vidéo…" (news.hamidun.com), section
  "Les trois techniques": the kernel gathers the selected key/value blocks
  by index, which is why the mask is also emitted as per-row index lists.

* the same AB-Attention page, section "Les trois techniques", second
  technique (SIP): sampled key blocks with inverse-probability logit
  offsets (``oracle.sip``).
* the same section, third technique: key groups of 4 tokens gathered by
  index into full tiles (``oracle.fine``).
* "SQuad: Sub-Quadratic Attention Distillation for Efficient Video
  Generation", section "Methodology: SQuad", item "1. SQuad-Attention
  Operator": the two-pass operator (``oracle.squad``).

Readings adopted where the pages are silent or garbled are listed in the
module docstrings of ``oracle.nabla``, ``oracle.sip``, ``oracle.fine`` and
``oracle.squad``.
"""
from .nabla import (  # noqa: F401
    Geometry,
    bf16_bits_to_f64,
    tile_reorder,
    tile_unreorder,
    block_mean_pool,
    pooled_score_map,
    cdf_select_row,
    cdf_select,
    sta_mask,
    build_block_mask,
    mask_to_lists,
    masked_attention,
    masked_attention_backward,
    masked_attention_backward_blocks,
    dense_attention,
    kept_pair_flops,
)
from .squad import squad_attention, squad_flops  # noqa: F401
from .sip import inclusion_probabilities, inclusion_probabilities_row, sip_attention, sip_sample  # noqa: F401
from .fine import build_fine_mask, fine_masked_attention, fine_score_map, kept_mass  # noqa: F401
