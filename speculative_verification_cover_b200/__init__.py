"""B200-native single-pass verification step for masked-diffusion speculative and
revocable decoding: dual-view (cache-override) attention with d_in/d_out,
fused vocabulary verification, stability-score seed selection and
KEEP/REPLACE/REMASK decisions, as sm_100a CUDA kernels behind a C ABI.

`speculative_verification_cover_b200.dd` binds the C ABI (libdd.so);
`speculative_verification_cover_b200.workloads` draws seeded synthetic inputs.
"""
