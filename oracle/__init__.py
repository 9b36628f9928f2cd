"""Plain fp64 CPU oracle for the spatial-temporal attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this
package; only the tests, the smoke check and the benchmark's CPU-baseline leg
call it.  It shares no code with the CUDA path: only the seeded input
generators in ``synth`` serve both.

Every function restates, in float64 numpy, what the pages define:

* attention   -- softmax(Q K^T * scale) V per unit, two-pass, no online
                 rescaling; spatial units are (b, t, head) over the S tokens
                 of a frame, temporal units are (b, s, head) over the T frames
                 of a token (ScaleFusion review, section "三、技术架构", layer
                 table and the spatial-temporal independence formulas).
* merge       -- log-sum-exp combination of KV-chunk partials, the step that
                 ring attention and SwiftFusion's Torus attention rely on
                 (SwiftFusion summary, Methodology 2 "Torus Attention").
* relayout    -- the all-to-all between the spatially sharded layout
                 [B,T,S/P,C] and the temporally sharded layout [B,T/P,S,C],
                 including the [B,N_T,N_S,T/N_T,S/N_S/P,C] slice layouts of
                 the intra-layer schedule (ScaleFusion review, section
                 "四、核心创新", intra-layer algorithm and pseudo-code), and the
                 Ulysses sequence<->head exchange (CoCoDiff article, Ulysses
                 section).
* rmsnorm     -- per-head RMSNorm on Q and K (CoCoDiff article, "V-First"
                 section).
* rope        -- rotary position embedding of Q and K after the RMSNorm
                 (CoCoDiff article, "V-First" section).
* vmajor      -- per-token L1 change of V against the previous step, the
                 threshold mask, the ascending list of active tokens and the
                 cache update (CoCoDiff article, "V-Major" section).

Each pin of these functions lives in ``tests/test_oracle_*.py``.
"""
from .attention import attention, spatial, temporal, merge_chunks, frames_view
from .relayout import (st_x_rows, st_y_rows, st_relayout, seq_head_relayout,
                       st_logical_from_x, st_logical_from_y, st_row_pairs, seq_head_row_pairs)
from .rmsnorm import rmsnorm_heads
from .rope import rope_angles, rope_table, rope_heads
from .vmajor import l1_change, change_mask, compact, scatter_rows, pack_rows, tau_for_fraction

__all__ = [
    "attention", "spatial", "temporal", "merge_chunks", "frames_view",
    "st_x_rows", "st_y_rows", "st_relayout", "seq_head_relayout",
    "st_logical_from_x", "st_logical_from_y", "st_row_pairs", "seq_head_row_pairs",
    "rmsnorm_heads", "rope_angles", "rope_table", "rope_heads",
    "l1_change", "change_mask", "compact", "scatter_rows", "pack_rows",
    "tau_for_fraction",
]
