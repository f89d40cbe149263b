"""HeadQ decode attention for NVIDIA B200 (sm_100a).

HeadQ ("HeadQ: Model-Visible Distortion and Score-Space Correction for KV-Cache
Quantization") stores each cached key as a 2-bit base code plus a low-rank
side code in a calibration-learned query basis and reads it back with an
additive logit correction.  The compute lives in ``libheadq.so`` (CUDA C-ABI,
``include/headq.h``); :mod:`.headq` is its thin Python binding.
"""
