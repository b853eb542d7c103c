"""fp64 CPU oracle for the MuonClip step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product (the C-ABI library and its Python binding) never calls it, and it
shares no code with the CUDA path.

Every function here is a plain, slow restatement of what the pages define,
in float64, with a matrix product as the only library primitive:

* ``oracle.muon``  -- momentum, Nesterov lookahead, orientation, Frobenius
  normalisation, quintic Newton-Schulz, RMS-matching scale, decoupled decay;
  the NorMuon per-row normalisation.
* ``oracle.qk``    -- per-head causal max logit S_max and the QK-Clip rescale.

Pins (tests/test_oracle_pins.py) tie each function to something other than
itself: the odd-polynomial/SVD identity, numbers the pages print, brute force
on tiny inputs, limits with a textbook answer, and a third-party optimizer.
"""
from .muon import (phi, phi_iter, phi_schedule, newton_schulz, muon_step, muon_step_many,  # noqa: F401
                   normuon_rows, normuon_step, minimax_odd_quintic, polar_express_schedule)
from .qk import (qk_max_logit, qk_max_logit_bruteforce, qk_clip, qk_clip_slices, mla_max_logit,  # noqa: F401
                 mla_slices, round_bf16)
