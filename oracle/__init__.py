"""CPU oracle for the Hiera mask-unit windowed block and the Hiera-B+ backbone.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may.
It shares no code with the CUDA library; the only common module is the seeded
input generator ``mask_unit_windowed_b200.synthetic``, which draws numbers and
holds none of the block's arithmetic.

Everything is float64 numpy. A library matmul / einsum / erf serves as a step;
there is no blocking, fusion or reordering beyond the definition.

Two independent formulations:
  * ``unrolled`` (formulation U) follows the "Phase 4: Hiera Backbone MLX Port"
    plan: tokens in [B, N, C], Unroll once after the patch embedding, mask-unit
    windows and pools taken on the unrolled token axis, Reroll at stage ends.
  * ``spatial`` (formulation S) restates the same network on NHWC grids: windows
    are square tiles, pooling is a 2x2 spatial max-pool, global attention is over
    the whole grid. It never forms the unrolled order.

Pins (see tests/test_oracle_*.py): Unroll/Reroll are inverse permutations;
q_stride 1 pools to the identity; one window of N tokens equals global attention;
the stage shapes the plan fixes; brute-force per-query loops on tiny grids;
U equals Reroll of S's features; closed forms for LayerNorm, softmax, GELU and an
all-zero block; equivariance under in-window token permutations.

Parity unpinned: the exact intermediate token layout of timm's Unroll (no timm
source or golden fixtures are available); the NHWC features do not depend on it.
"""
