"""CPU oracle for the NeRF renderer, its march scene functions and its training step: plain, slow, fp64 numpy.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, links or calls
this package; only the tests, the smoke check of the build entry point and the
CPU-baseline leg of the benchmark do. It shares no code with the CUDA library:
inputs come from ``nerf_inputs`` (a module that holds none
of the method's arithmetic), and every function here is written from the pages'
definitions, each citing the page and section it follows.

Page names used in citations:
  "NeRF page"      = "Spatial Intelligence - Part 1: NeRF" (halannhile.github.io)
  "Instant-NGP notebook" = "Instant-NGP - Visual Experiments (a 2D multiresolution
                     hash grid)" (triet4p.github.io latent-anything notebook 05)
  "KiloNeRF page"  = "KiloNeRF: Speeding up Neural Radiance Fields with Thousands
                     of Tiny MLPs" (codewithpapers.app metadata, abstract)

Precision: arithmetic is fp64 except where a floating-point value decides an
integer or a sample position (ray directions, sample positions t, points x,
voxel/cell/hash-corner choice, inverse-CDF bin choice). Those steps are
evaluated in IEEE fp32 with a fixed operation order, written out below, so that
the CUDA path can take the same decisions bit for bit.

Parity status: every function is pinned by tests under tests/ (closed forms,
printed values from the pages, invariants, brute force on tiny inputs); see the
"pins" column of the design notes. None is "parity unpinned".
"""
