"""CPU oracle for the FP4 micro-scaled linear layer -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct restatement of what the
method computes, written from the pages' descriptions:

* "Quartet: Native FP4 Training Can Be Optimal for Large Language Models"
  (MXFP4 training: Hadamard-32 + QuEST forward, randomized Hadamard + SR
  backward, the clip-mask epilogue);
* "Quartet II: Accurate LLM Pre-Training in NVFP4 by Improved Unbiased
  Gradient Estimation" (NVFP4 format, NVIDIA-style SR, Four-Over-Six,
  MS-EDEN and its post hoc range alignment);
* "Bridging the Gap Between Promise and Performance for Microscaling FP4
  Quantization" (MXFP4/NVFP4 formats, the E2M1 dead zone, Lemma 1).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The product path
(the CUDA library and its Python binding) never imports, calls or links
anything here, and nothing here imports the product path.

Arithmetic contract (shared by definition, not by code, with the GPU path):
quantizer arithmetic is IEEE fp32 with round-to-nearest-even on every
operation (numpy float32 ops, no fused multiply-add), division is correctly
rounded, sums are fixed pairwise trees (float64 in the MSE search's
tensor-scale step), maxima are exact; GEMM references are fp64.
"""
