"""Float64 CPU oracle for calibrated block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
The product path (``calibrated_block_sparse_calib_b200`` and ``libcalibatt.so``) never
imports, links or executes anything here, and this package imports nothing from it.

Sources.  The method is stated only in prose on five web pages; there is no code,
equation, table or worked example to copy.  Citations use these tags:

  [zh]  "Accelerating Text-to-Video Generation with Calibrated Sparse Attention"
        (gist.science, Chinese) -- technical summary, sections 2.1 / 2.2A / 2.2B
  [de]  same paper (gist.science, German) -- "Technische Zusammenfassung" §2A / §2B
  [pt]  same paper (gist.science, Portuguese) -- "Resumo técnico" §2A / §2B
  [fr]  same paper (gist.science, French) -- "Résumé technique" §2.A / §2.B / §2.C
  [AdaSpa] "Training-free and Adaptive Sparse Attention for Efficient Long Video
        Generation" (PKU-DAIR summary page) -- §2 "方法"

Every function states which passage it follows and, where the pages leave a step
open, which reading it takes.  Pins (tests/test_oracle_*.py) check each function
against closed forms, invariants, brute force and library routines; no function
here is "parity unpinned".
"""
from .calibatt_ref import (  # noqa: F401
    logits, row_lse, block_energy, energy_mean, quantize_row, select_row, select_mask,
    aggregate_masks, mask_to_csr, csr_to_intervals, intervals_to_csr, build_schedule, anchor_rows,
    anchor_index_of_token, anchor_token, repeat_similarity, repeat_flags,
    sparse_attention, sparse_attention_repeat, ceil_log2,
)
