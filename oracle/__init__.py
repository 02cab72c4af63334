"""CPU oracle for the QLoRA NF4 + LoRA quantized linear.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain, obviously
correct statement of what the CUDA library computes. Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. The product path never calls it, and it
never imports the product package: the two share no code, tables or
constants.

Sources (cited by page title and section throughout):

* «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나» (iq-universe blog) —
  § "QLoRA의 수식: 두 항의 결합" (the forward formula), § "명제 1 · QLoRA
  Backward Unbiasedness" (gradients only into A and B), § "메모리 회계"
  (4.5 and 4.13 bits/param, the double-quantization formula and its
  s_max/256 bound).
* "48GB GPU Fine-Tuning a 65B Model: Where QLoRA Saves GPU Memory" —
  § "Quantization Keeps the Patterns and Reduces Bits per Number" (blocks of
  64, absmax scale, divide-then-nearest-level, normal-quantile levels with an
  exact zero, 8-bit scale codes, bf16 restore), § "QLoRA Puts the Two
  Methods in Different Places" (forward and backward in words),
  § "LoRA Freezes the Original Weights ..." (B = 0 start).
* "QLoRA: Efficient Finetuning of Quantized LLMs" (tellworld summary) —
  § "How it works" (NF4 for normally distributed weights).

Modules
-------
``nf4``     codebook, blockwise absmax, encode, pack, double quantization,
            dequantization (numpy, IEEE fp32 steps as defined).
``linear``  forward and backward of the quantized linear in fp64.
``brute``   literal pure-Python loops for tiny inputs (pins ``nf4``).
``bf16``    float32 <-> bfloat16 round-to-nearest-even bit helpers.

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against something other than itself (closed forms, brute force, finite
differences, identities). The codebook's agreement with any externally
published NF4 table is not pinned by the pages ("parity unpinned" for that
comparison only; the construction itself is pinned by the quantile identity).
"""

from . import bf16, nf4, linear, brute  # noqa: F401
