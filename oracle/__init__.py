"""Float64 CPU oracle for the mixed-precision MoE expert path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA path (``mixed_precision_expert_b200``); the
two meet only in the seeded input generators of ``synth``.

What it computes, each module citing the passage it follows (PagedWeight =
"PagedWeight: Efficient MoE LLM Serving with Dynamic Quality-Aware Weight
Quantization", llmdb.app summary page):

* ``allocate``  -- the budgeted precision problem of PagedWeight,
  "Quality-Aware Quantization" (min sum_e p_e L(b_e) s.t. sum_e b_e W_e <= B,
  b_e in {3,4,8} from "Code Illustration" bit_options), solved exactly by a
  dynamic program over budget units.
* ``quantize``  -- PagedWeight, "Implementation Details", quantization scheme:
  Q(w) = round(w/s) s, s = max|w| / (2^(b-1) - 1), one scale per expert.
* ``layout``    -- the bit-width-specific page format (PagedWeight, "Dynamic
  Paging": experts stored in pages of 8-, 4- or 3-bit width); the exact byte
  layout is this project's own definition.
* ``pages``     -- the page allocator and page table (PagedWeight,
  "Implementation Details", memory management: a page table maps expert IDs
  to physical pages).
* ``route``     -- token-to-expert bucketing for the forward pass (PagedWeight,
  "Dynamic Paging": the router decides which experts a pass needs).
* ``compensate`` -- dynamic error compensation of salient input channels
  (DecDEC summary, 3.1-3.2 and Figure 4): (W^ + R (.) M) x with R = W - W^
  and M keeping the channels of largest |x|.
* ``prefix``    -- the prefix-compatible variant: a nested grid (the b-bit
  code is the top b bits of the 8-bit one) stored in layers, so a width
  change drops or adds layers instead of re-encoding.
* ``ffn``       -- dequantize-then-multiply expert FFN (PagedWeight, "Dynamic
  Paging": fetch pages, dequantize on the fly; DecDEC summary, 2.2: weight-only
  quantization dequantizes before multiplying with full-precision
  activations), SwiGLU form, top-k weighted combine.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, hand-worked values, exact rational arithmetic or brute
force; none is "parity unpinned".
"""
