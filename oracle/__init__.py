"""CPU oracle for the W4A4 quantized linear layer (test infrastructure only).

This package is the plain, slow, obviously-correct statement of what the GPU path
computes, written from the pages' definitions in float64 (float32 where a rule is
defined as a float32 operation so that the GPU can take the same integer decision).
It shares no code with the CUDA library and never imports it.  Only the tests, the
package's ``smoke()`` check and the CPU-baseline leg of ``bench.py`` may import it;
the product path must never route through it.

Modules
-------
formats   E2M1 / E8M0 / E4M3 / UE5M3 / INT4 codecs (MXCode, Table 1; OCP MX formats).
mx        Activation/weight quantizers: E8M0-B32, E4M3-B16 + FP32 tensor scale, INT4 g128.
gemm      Block-scaled W4A4 GEMM reference and the per-element tolerance scale.
prquant   PRQuant offline column selection (optionally with the E8M0-W block-scale search),
          permutation, tail residual, the augmented activation and GEMM.
vq        MXCode VQ: PreScale E4M3-B16 scales, per-QBlock FP4 codebooks, index assignment;
          PostScale (one scale per codebook) and PreScale+ (scale indices into a scale codebook).
hadamard  Block-32 Walsh-Hadamard of the activations ahead of the MXFP4 quantizer (CodeQuant had).
moe       Top-k routing and the grouped SwiGLU expert FFN with cluster-codebook weights.
int4bsr   MosaicQuant-style INT4 dense base + block-sparse INT4 residual.

Parity unpinned: the k-means codebook quality (data synthesis only), and the realism of
the synthetic router; neither changes what the path computes given its inputs.
"""
