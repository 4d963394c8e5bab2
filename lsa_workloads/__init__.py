"""Seeded synthetic workloads for the LSA decode step.

This module draws random inputs and lays them out; it performs none of the
method's arithmetic (no scores, gates, selections or attention).  It serves
the tests, the smoke check and the benchmark alike.

Random numbers: numpy PCG64, one independent stream per (workload seed,
stream id, block), so any block can be regenerated on its own.  bf16 values are
fp32 draws rounded to nearest-even and are handed around as uint16 bit patterns.

Workloads (the arXiv 2606.09079 pages give no model dimensions; the chunk size,
head shapes, latent width and top-k size below are this build's workload
definition):

  decode_16k_b1_h16        batch 1, 16,384-token context (256 chunks); NMI 8x64;
                           Lightning indexer 8x64, top-k 512; attention 16 heads
                           over one KV head, K and V rows of 128 each.
  decode_128k_b8_mla       batch 8, 131,072 tokens (2,048 chunks); NMI 64x128;
                           indexer 64x128, top-k 2048; 128 heads over one latent
                           KV row of 576 (first 512 columns are V).
  decode_512k_b1_mla_cold  batch 1, 524,288 tokens, shapes as above; chunks before
                           the recent window live in pinned host memory.
  decode_ragged_b32_mla    32 sequences, context log-uniform in [16K, 512K]
                           rounded to 64, per-sequence pass rate U[5%, 25%].
  label_vote_128k_l32      32 layers x 64 steps x 2,048 chunk scores.
"""
from .generate import (  # noqa: F401
    CHUNK, WINDOW, STEPS, Workload, WORKLOADS, LABEL_VOTE, workload,
    to_bf16_bits, bf16_bits_to_f32, normal_bf16,
    nmi_inputs, next_window_plant, resident_layout, cold_layout, chunk_rows, kv_pools, host_pool,
    step_inputs, label_vote_scores, redraw_slice, nudge_bits,
    encoder_inputs, ENCODER_D_MODEL, ENCODER_RANK,
)
