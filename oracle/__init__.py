"""CPU oracle for the SSD chunked scan — TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the bench's CPU-baseline leg use
this package.  The GPU library never imports it, and it imports nothing from the
GPU library: the two share no code, only the seeded input generator in
`harness/`, which holds none of the scan's arithmetic.

Sources followed (page titles as they appear on the web):
* "SSDi8: Accurate and Efficient 8-bit Quantization for State Space Duality"
  (ICLR 2026 paper notes) — the five SSD sub-modules (section "overall
  framework"), eq. 4 and the sparsity-aware reconstruction (key design 1), the
  INT32→INT8 state requantisation and eq. 6 (key design 2), the per-G / per-(H,P)
  quantisation axes (key design 3), symmetric static PTQ (training strategy).
* The recurrence the chunked algorithm factorises:
  h_t = exp(dt_t·A)·h_{t-1} + dt_t·x_t B_tᵀ,  y_t = C_t·h_t + D·x_t.

Modules:
* `ssd_fp64`  — fp64 sequential recurrence, quadratic "attention form" brute
  force, fp64 chunked form (ChunkCumsum … ChunkScan); calibration.
* `ssd_w8a8`  — the integer W8A8 pipeline with its fp32 prelude specified op by
  op, so that every integer it produces is reproducible bit for bit.
* `study_xscaled` — quantisation error of Q(X_scaled) against Q(X)⊙LUT_state
  (the comparison of key design 1's appendix claim), measured on given inputs.

Parity status per function is listed in each module's docstring.
"""
