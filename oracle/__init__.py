"""CPU oracle for MLA weight-absorbed decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (``mla_latent_kv_34_b200``) never imports it and shares no code with it;
the two meet only in the seeded input generator ``mla_inputs``.

Sources (the pages describing DeepSeek-V2 Multi-head Latent Attention):
  * "DeepSeek-V2/V3: 大模型的两张账" (chenyuan1125.github.io), section
    "第一张账": c_t^KV = W^DKV h_t; k_t^C = W^UK c_t^KV, v_t^C = W^UV c_t^KV;
    the cache holds only c_t^KV and the shared RoPE key k_t^R; attention
    matches the concatenation [content; position] of query and key; W^UK can be
    absorbed into the query side and W^UV applied after aggregating in latent
    space; the official inference code names the "naive" and "absorb" paths.
  * "DeepSeek-V2 ... MLA" explainer (xinfinite.net), sections 2.2.1.1 (joint
    KV compression and its up-projections), 2.2.2 (decoupled RoPE: per-head
    q^R, one shared k^R, the RoPE'd key part is cached; S = Q^T R_m^T R_n K),
    and the cache size (d_c + d_h^R) l, "GQA with 2.25 groups".
  * DeepSeek-V2 reading notes (chenshi221.pages.dev), "Method 1. MLA": the KV
    cache table (MHA 2 n_h d_h l, GQA 2 n_g d_h l, MQA 2 d_h l, MLA ~9/2 d_h l).

Modules:
  naive   -- fp64 naive decode (explicit k^C, v^C per head; textbook softmax),
             the fp64 absorbed form, split-KV partials and their LSE merge,
             RoPE, cache-footprint formulas, and the query-side up-projections
             q^C = W^UQ c^Q, q^R = W^QR c^Q of the compressed query.
  append  -- bit-exact emulation of the cache append in the kernel's fp32
             arithmetic (RoPE table rounded to fp32; separate multiplies and
             adds; round-to-nearest-even to bf16).

Readings taken where the pages are silent (each is a documented choice):
  * softmax scale 1/sqrt(d_h + d_h^R) = 1/sqrt(192);
  * RoPE pairs adjacent dims (2i, 2i+1), theta_i = base^(-2i/d_h^R), base 10000;
  * the key at cache index t has position t; query j of a step with n_q new
    tokens has position L_b - n_q + j and sees keys t <= L_b - n_q + j.
  * q^R is an up-projection of the compressed query c^Q, like q^C (its formula
    is lost on the pages).
"""
