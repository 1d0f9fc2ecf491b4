"""CPU oracle for the vecset SDF decoder and its lightning-decoder procedures.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the CUDA path computes, in float64 numpy.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it.  It shares no code with ``neural_sdf_volume_b200`` (the CUDA path), and the
CUDA path never imports it; the only common module is ``workloads`` (seeded
input generators, no decoder arithmetic).

Sources (FlashVDM, "Unleashing Vecset Diffusion Model for Fast Shape
Generation", as summarised on the aipaper.cc page and the techwalker.com
article):

* vecset decoder: cross-attention from query points to the latent token set,
  then the SDF at arbitrary points (section 3, foundational concepts);
* hierarchical volume decoding with tSDF-style near-surface selection and one
  dilation (section 4.1, item 1 and its corner-case notes);
* adaptive KV selection with sub-volumes, random probe queries, attention
  scores and Top-K tokens (section 4.1, item 2; "packing" note);
* efficient decoder: narrower width, smaller MLP ratio, fewer LayerNorms
  (section 4.1, item 3).

Modules
-------
``decoder``    Fourier embedding, LayerNorm, GELU, K/V projection, multi-head
               cross-attention (dense or over a token subset), MLP, SDF head,
               analytic sphere term.
``hierarchy``  cell-centred grids, boundary marking, dilation, compaction,
               inherit-fill and the coarse-to-fine level loop.
``adaptive``   SplitMix64 probe ranking, sub-volume binning, probe scores,
               Top-K and the adaptive fine-level decode.

Parity pins live in ``tests/test_oracle_*.py``.  Where the pages leave a
step open, the reading taken is stated in the docstring of the function that
implements it.
"""
