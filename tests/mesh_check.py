"""The step-size controller's chain over a recorded mesh, checked against the
oracle's view of that mesh (oracle.step_errors: each step's scaled error and
the PI factor accepting it gives).

The recorder proposes h_prop, takes min(h_prop, distance to the next stop),
and after an accepted step proposes fac * h_prop (h_prop unclipped; fac capped
at 1 right after a rejection); a rejection multiplies h_prop by a factor
< 1 and retries.  A mesh holds accepted steps only, so along trajectory i:
- a step that does not end on a stop (a save time or t1) equals the proposal
  the chain predicts, unless rejections shortened it (then it is shorter);
- a step that ends on a stop is at most the proposal.
The chain restarts from every step that does not end on a stop."""
import numpy as np


def controller_chain(h, nsteps, save_idx, nreject, fac, tol, all_devs=None):
    """Walk every trajectory's chain.  tol: the relative tolerance of one
    factor, a scalar or per step [n][smax] (tol[i, s] for the factor after
    step s); a prediction carried over hidden steps takes the sum of its
    factors' tolerances.  Returns (dev, short, bad): dev [n] the largest
    |h_s / h_pred - 1| / tol_pred over predicted steps that do not end on a
    stop and were not shortened, short [n] the steps shortened by more than
    their tolerance (each needs at least one rejection), bad [n] the steps
    longer than the prediction by more than their tolerance (none for a
    recorder that follows the chain).  all_devs, a list, receives every such
    step's signed h_s / h_pred - 1 (rounding noise is centred on 0; a wrong
    controller constant shifts them all)."""
    n = len(nsteps)
    tarr = np.broadcast_to(np.asarray(tol, np.float64), np.shape(fac))
    dev = np.zeros(n)
    short = np.zeros(n, np.int64)
    bad = np.zeros(n, np.int64)
    for i in range(n):
        ns = int(nsteps[i])
        stops = set(int(k) for k in np.atleast_1d(save_idx[i])) | {ns}
        hp = alt = None  # predicted proposal; alt: the same with the cap after a hidden rejection
        tp = 0.0         # its tolerance
        cap = False
        for s in range(ns):
            landed = (s + 1) in stops
            hs = float(h[i, s])
            shortened = False
            if hp is None:
                if not landed:
                    hp, tp = hs, 0.0
            elif landed:
                if hs > hp * (1 + tp):
                    bad[i] += 1
            else:
                r = hs / hp
                if alt is not None and abs(hs / alt - 1) <= tp < abs(r - 1):
                    # a rejection before the last landing step capped this factor
                    r = hs / alt
                    short[i] += 1
                if r < 1 - tp:
                    short[i] += 1
                    shortened = True
                else:
                    dev[i] = max(dev[i], abs(r - 1) / tp if tp > 0 else (0.0 if r == 1 else np.inf))
                    if all_devs is not None:
                        all_devs.append(r - 1)
                    if r > 1 + tp:
                        bad[i] += 1
                hp, tp = hs, 0.0
            alt = None
            if hp is not None:
                f = float(fac[i, s])
                if cap or shortened:
                    f = min(f, 1.0)
                elif landed:
                    alt = min(f, 1.0) * hp
                cap = False
                hp = f * hp
                tp += float(tarr[i, s])
    return dev, short, bad
