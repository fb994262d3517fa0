"""CPU oracle for the routed-expert MoE FFN with MXFP4 weights and FP8 activations.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything under ``oracle/``; it is used by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / reference leg of
``bench.py``.  It shares no code with the CUDA path (``fp8_block_scaled_pow2_b200``);
both receive their inputs from the separate ``synth`` module.

The oracle is plain, slow and written to be checked by eye against the source
pages.  Floating-point arithmetic is float64 except where a float decides an
integer (a quantised code or a power-of-two exponent): there the decision is
taken in float32, the precision the kernels use, because the pages do not fix
one.  Library primitives used as steps: numpy matmul (float64), stable sort.

Modules and the passages they follow:
  formats  -- E2M1 / E8M0 / E4M3 / bf16 decoding, E4M3 rounding
              ("DeepSeek-V4-Flash-SI" model card, 架构特性 / 低精度计算;
               "DeepSeek-V4-Pro-0813-nvfp4-DSpark" walkthrough, 关于 MXFP4 的无损种子)
  quant    -- online FP8 E4M3 activation quantisation, one power-of-two scale
              per 128 elements (DeepSeek-V4-Flash-SI, 低精度计算 and 模型训练 table)
  route    -- sqrtsoftplus top-k routing with route scale 1.5, and the hash routing
              of the first layers read as a token-id -> experts table lookup
              (DeepSeek-V4-Flash-SI, 架构特性, Mixture of Experts paragraph)
  permute  -- grouping routed (token, slot) pairs by expert
  ffn      -- grouped expert GEMMs w1/w3 and w2, SwiGLU with the +-10 clamp,
              weighted combine, the W4AFP8 variant
              ("DeepSeek-V4-Flash-0731-W4AFP8-mt" model card, 量化方式 / 权重约定),
              the FP8 [128, 128]-block shared expert (DeepSeek-V4-Pro-0813-nvfp4-DSpark,
              只量化专家; DeepSeek-V4-Flash-SI, 模型训练) and the PTPC-FP8 path
              ("DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough, 核心参数)
  repack   -- MXFP4 -> NVFP4 (DeepSeek-V4-Pro-0813-nvfp4-DSpark, 阶段三 storage table),
              MXFP4 -> symmetric INT4 group 128 (W4AFP8-mt, 量化方式 / 权重约定) and
              MXFP4 -> FP8 E4M3 with [128, 128] block scales (nvfp4-DSpark, 关于 MXFP4 的无损种子)

Parity pins (tests/test_oracle_*.py) tie each function to something other than
itself: the E2M1 value set, exhaustive E8M0 / E4M3 code tables, hand-derived
rounding cases, closed forms, brute force on tiny inputs, the INT4 shape
example of the W4AFP8 card and the lossless property of the NVFP4 cast.
Where the pages leave a point open the oracle takes the plainest reading and
says so at the function.  Six readings are "parity unpinned" because no page
fixes them: the nibble order inside a byte (element 2i in the low nibble), the
exact INT4 scale rule (amax / 7), the PTPC-FP8 scale rule (amax / 448), the
normalisation of the routing weights before the 1.5 scale (flag route_norm),
the clamp of both the gate and the up projection to +-10 before
silu(g) * u, and hash routing as a lookup in a caller-supplied table (the
page names hash routing by token ID but gives no hash).
"""
