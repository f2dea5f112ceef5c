"""CPU oracle for the QLoRA NF4 frozen-base linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import or run anything here.
The CUDA library never calls this code and shares no code, table or constant
with it; both sides get their inputs from the seeded generators in ``synth/``.

What it computes, step by step, in plain NumPy/SciPy (fp64 wherever the method
does not fix a precision; explicit float32 rounding where the method is defined
on 32-bit values):

* ``nf4.nf4_levels``  -- the 16 NormalFloat levels.  Sources: "QLoRA"
  (ai360xpert.com), How It Works 1; "QLoRA: Efficient Finetuning of Quantized
  LLMs" (crackai.dev), How It Works 1 (levels at normal quantiles, the same
  probability mass in every bin); "QLoRA"
  (ozercemkelahmet.com), How it works -- Why NormalFloat.
* ``nf4.quantize``    -- blockwise absmax (64 values), nearest level, two codes
  per byte; then the 8-bit double quantization of the block constants in groups
  of 256 with one fp32 constant per group.  Sources: ozercemkelahmet.com, How it
  works, Steps 1-3 and "A worked example"; crackai.dev, How It Works 2.
* ``nf4.dequantize``  -- level times reconstructed block constant, rounded to the
  bf16 compute type.  Sources: ozercemkelahmet.com, Overview and Step 5;
  "QLoRA" essay (fanfani.net), section "The crucial split".
* ``linear.forward`` / ``linear.backward`` -- Y = X deq(W)^T + s (X A) B and its
  gradients for X, A, B (W frozen), accumulated in fp64.  Sources:
  ozercemkelahmet.com, How it works, Steps 5-6.
* ``linear.merge_weight`` -- the adapter folded into a 16-bit weight,
  bf16(W_base + s (A B)^T), rounded once from the fp64 sum
  (``nf4.f64_to_bf16_rn``).  Sources: ozercemkelahmet.com, How it works, Step 8,
  section "Merging after QLoRA", and its FAQ on merging.
* ``nf4.quantize_single_level`` / ``nf4.dequantize_single_level`` -- Steps 1-2
  without Step 3: the same codes, the block constants kept in fp32 (half a bit
  per weight).  Source: ozercemkelahmet.com, How it works, Step 2.
* ``linear.forward_dropout`` / ``linear.backward_dropout`` /
  ``linear.accumulate_grads`` -- inverted dropout of the adapter input with a
  caller-drawn keep mask, and dA / dB summed over micro-batches.  Sources:
  ozercemkelahmet.com, "A code example with common libraries" (lora_dropout),
  "Training arguments" (gradient_accumulation_steps) and "Reading the memory
  profile".

Readings taken where the pages are silent (each one is listed with its reason in
the design notes of the repository):

* table: asymmetric halves (8 positive, 7 negative levels, one exact zero),
  quantiles evenly spaced in [0.5, P_MAX] with P_MAX = (1 - 1/32 + 1 - 1/30)/2,
  normalised to [-1, 1].  The exact P_MAX is a named constant the pages do not
  print: *parity unpinned by the pages* for that constant; the table is pinned
  by its invariants (16 monotone levels, exact 0 and +-1, equal mass per bin).
* normalisation ``xn = RN32(w / absmax)``; nearest level in exact arithmetic,
  ties to the lower index; all-zero block -> code of the zero level.
* double quantization: unsigned linear 8-bit code of the (non-negative) block
  absmax, ``step = RN32(c_g / 255)`` with ``c_g`` the group maximum,
  ``q8 = min(255, rint_even(RN32(a_b / step)))``.  Pinned by the closed-form
  storage overhead and the quantization error bound, not by printed values.
* packing: element 2j in the low nibble of byte j.
"""
