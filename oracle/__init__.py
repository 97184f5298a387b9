"""CPU oracle for the SVDQuant W4A4 (NVFP4) linear layer -- TEST INFRASTRUCTURE.

This package is a plain, slow, deliberately simple restatement of what the
layer computes, in numpy (float64 wherever the method does floating point
and the format does not fix the precision).  It exists to check the CUDA
path, never to serve it: only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / reference leg of `bench.py` may import it.  It shares no
code with `w4a4_rank_corrected_b200` and imports nothing from it.

Sources (page title -- section):
  * "SVDQuant: 4-Bit Quantization Powers 12B Flux on a 16GB 4090 GPU with 3x
    Speedup" (Hacker News thread) -- outlier absorption by a low-rank
    decomposition combined with smoothing; "a LoRA to reconstruct outliers".
  * "Bringing Nunchaku 4-bit diffusion inference to Diffusers" (Vietnamese,
    Russian and Korean renderings) -- "Background: SVDQuant and Nunchaku":
    activation outliers are moved into the weights, the hardest part of
    each weight is a small 16-bit low-rank branch, the residual is
    quantized to 4 bit; the hardware table: svdq_w4a4 in NVFP4 on Blackwell.

Parity status per function is written in each docstring.  Every reading of
a point the pages leave open is listed in the module docstring of
`oracle.svdq`.
"""
