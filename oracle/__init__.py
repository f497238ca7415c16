"""Plain fp64 CPU oracle for the Wan DiT hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or call it.  It shares no
code, header, table or helper with the CUDA library; both sides only receive
the same seeded input arrays.

Every function is written from the text of the source pages and cites the
passage it follows.  The pages are:

* "Wan2.2 source reading" -- the blog post "動画生成の勘定を明らかにする：
  Wan2.2 ソースコード精読" (blog.leeguoo.com), cited by chapter and section;
* "Wan paper explainer" -- "論文解説: Wan - 大規模オープンソース動画生成
  モデルのアーキテクチャと訓練" (0h-n0.github.io), cited by section;
* "Long-video survey" -- the atlascloud.ai long-video generation blog, cited
  by section.

Modules:

* ``grid``      -- latent shape and token grid arithmetic;
* ``rope``      -- 3D rotary position embedding (t/h/w bands);
* ``attention`` -- softmax self-attention and length-masked cross-attention;
* ``schedule``  -- shifted sigma schedule and timestep scale;
* ``step``      -- classifier-free-guidance combine and Euler flow step;
* ``block``     -- AdaLN modulate, QK-Norm + RoPE, gated residual around the
  attention;
* ``unipc``     -- the UniPC order-2 predictor-corrector sampler step (the
  pages give no coefficients: written from the published UniPC order
  conditions, pinned by exactness and convergence order).

Pins (tests/test_oracle_*.py) tie each function to numbers the pages print,
closed forms and brute force.  The one part the pages do not fix numerically
is the RoPE frequency base and pair layout: the pages print no rotated value,
so the RoPE *values* are "parity unpinned" beyond the invariants the pages
state (translation invariance of q.k, identity at the origin, norm
preservation); the readings taken are listed in ``rope``'s docstring.
"""

from . import grid, rope, attention, schedule, step, block, unipc  # noqa: F401,E501
