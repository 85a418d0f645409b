"""Plain, slow, fp64 CPU oracle for few-bit KV-cache compression and decode attention.

This package is TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the product path (``bit_kv_cache_seeded_b200``)
never does, and the oracle imports nothing from the product. The two share no code, tables,
constants or helpers: the only thing both sides consume is the seeded input generator in
``kvq_inputs`` (random numbers and synthetic tensors, none of the method's arithmetic).

What it follows (cited by page title and section):

* "TurboQuant vs OSCAR vs EpiCache" (dothoosh.com), section "Quantization frontiers:
  TurboQuant and OSCAR": stage one rotates every vector at random so that its coordinates are
  close to independent Gaussians and applies a precomputed Lloyd-Max scalar quantizer per
  coordinate; stage two applies a 1-bit quantized Johnson-Lindenstrauss transform (QJL) to
  the residual, which gives an unbiased estimate of attention logits. The same section places
  the distortion within a small constant (about 2.7x) of the information-theoretic bound.
* Same page, section "KV-cache bottleneck": the bf16 KV-size arithmetic and the fact that each
  decode step streams the whole cache.
* "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", sections "CSA2" (a 512-dim
  latent shared by all heads) and "Numerics and hardware efficiency" (FP4 E2M1 with one scale
  per 16 channels); "DeepSeek-V4.1-Flash cuts KV cache to 890 bytes per token", FP4 bullet.
* "TaSQ 1-bit KV cache compression boosts batch sizes 14x": a 1-bit KV cache.

Modules:
  tables    -- Gaussian Lloyd-Max tables by fixed-point iteration, Sylvester-Hadamard matrix,
               FP8 E4M3 and FP4 E2M1 codecs (all from their definitions).
  codec     -- per-vector quantization (rotation, normalisation, Lloyd-Max code, residual,
               QJL sign sketch, bit-plane packing), the 1-bit variant and the FP4 variant.
  attention -- dequantisation and decode attention (original domain, two-pass softmax), the
               rotated-domain formulation, and the MLA-style latent attention.
  sizes     -- KV bytes-per-token arithmetic.

Parity unpinned: nothing in this package is left without a pin; the page-level quality claims
(3.5-bit neutrality, needle-in-a-haystack recall) need models and datasets and are not
computed here at all.
"""
