"""CPU oracle for the sink-window attention hot path — TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 NumPy restatements of what the method computes, written
from the source pages (the LongLive paper review "LongLive: Real-time
Interactive Long Video Generation" and the LoL review "LoL: Longer than Longer,
Scaling Video Generation to Hour"). Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package. The CUDA library never calls it and shares no code with it; the
only common code is the seeded input generator in ``swa_workloads``.

Modules
-------
rope       per-head frequency tables, LoL jitter, 2x2 pair rotation, 3D RoPE
window     frame-sink + short-window attended set and the cache slot map
attention  textbook multi-head attention and sink-window attention over frames
recache    projection + RMSNorm + RoPE of the cached frames at a prompt switch
fp8        OCP FP8 E4M3 encode/decode and per-(token, head) quantisation
stream     a frame-by-frame stream driver that keeps per-frame K/V history

Pins (tests run with ``-m "not gpu"``) tie each function to something other
than itself: closed forms, identities, brute force, library routines and the
constants the pages print. Parts with no such pin are listed as
"parity unpinned" below.

parity unpinned: none of the functions here; model-dependent quantities
(real K/V statistics, sink-collapse metrics) are outside this oracle.
"""
