"""CPU oracle for the TurboQuant hot path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 NumPy/SciPy restatement of what the method computes, used to
check the CUDA library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path never does, and this package never imports the product.

Sources (web pages; cited by title and section):

* R  -- "TurboQuant: Online Vector Quantization with Near-optimal Distortion Rate",
        paper review (sections Problem, Method, Validation, Results, Comparison,
        Limitations; Figure 3(a) caption).  The authority on the method.
* LK -- "TurboQuant Launch Kit" (LAUNCH.md): X thread posts 5/16 and 8/16,
        Show HN post (rotation modes, "codebooks are fixed at init").
* SQ -- SpectralQuant thread by @ashwingop, posts 2, 4, 5, 6 (eigenvector
        rotation, 4 signal dims, selective QJL, water-filling [5,3,2,2]).
* VZ -- "From dense vector to score-preserving code" (Online Compression
        Pipeline; Decode traffic per token).

Modules:

* :mod:`oracle.codebook`  -- Lloyd-Max codebooks for the post-rotation marginal
  (Beta on the sphere, or its Gaussian limit), cell moments, distortion D_b.
* :mod:`oracle.quantizer` -- TurboQuant-mse / -prod quantize, dequantize, the
  inner-product estimator, and the packed record format.
* :mod:`oracle.spectral`  -- SpectralQuant-style calibration, water-filling,
  per-dimension codebooks, quantize and estimator.
* :mod:`oracle.attention` -- decode attention (softmax(q.k_hat / sqrt(d)) v_hat)
  straight from the quantized records, and dense scores.
* :mod:`oracle.search`    -- exhaustive top-k by estimated inner product.
* :mod:`oracle.split`     -- outlier-channel split: independent TurboQuant instances
  on channel groups (online outlier detection, per-group quantize, summed estimates).
* :mod:`oracle.sweep`     -- inner-product distortion of the mse and prod variants by
  bit width (bias and total), on correlated query/key pairs.
* :mod:`oracle.serving`   -- paged-cache slots, and causal prefill attention over the
  quantized cache (append-then-attend is the quantize and decode steps in sequence).

Every function here is pinned by ``tests/test_oracle_*.py`` against closed forms,
printed values, brute force or library routines, except where its docstring says
"parity unpinned".
"""
