"""Writes closed_forms.json: hand-derived special cases of the OPD loss and its gradient.

The pages print no worked example, so these cases are derived by hand from the definitions
(reverse-KL d_v = q_v log(q_v/p_v), entry-wise clip min(d_v, c), hard-label CE on the target
argmax, the lambda mix, temperature dividing both logit sets).  Each case is small enough that
every quantity has a closed form in e = exp(1); this script evaluates those closed forms with the
``math`` module only (it calls neither the oracle nor the CUDA library).
Run:  python tests/golden/make_closed_forms.py
"""
import json
import math
import os

E = math.e


def case_clip_v2():
    # D = [0, 0], T = [1, 0], tau = 1, lambda = 0.5, c = 0.25.
    # q = (1/2, 1/2), p = (e/(1+e), 1/(1+e)).
    lam, c = 0.5, 0.25
    s0 = math.log((1 + E) / (2 * E))       # log q0 - log p0 (< 0)
    s1 = math.log((1 + E) / 2)             # log q1 - log p1 (> 0)
    d0, d1 = s0 / 2, s1 / 2                # d1 = 0.31 > c: entry 1 is clipped
    assert d0 < c < d1
    Kc = d0 + c
    rkl = d0 + d1
    ce = math.log(2)                       # y = argmax T = 0, q0 = 1/2
    L = lam * ce + (1 - lam) * Kc
    S = 0.5 * (s0 + 1)                     # only the unclipped entry 0 contributes
    g0 = lam * (0.5 - 1) + (1 - lam) * 0.5 * ((s0 + 1) - S)
    g1 = lam * 0.5 + (1 - lam) * 0.5 * (0 - S)
    return dict(name="clip_v2", D=[0.0, 0.0], T=[1.0, 0.0], tau=1.0, lam=lam, clip_c=c,
                loss=L, rkl=rkl, kc=Kc, ce=ce, grad=[g0, g1],
                derivation="q=(1/2,1/2), p=(e/(1+e),1/(1+e)); s0=log((1+e)/(2e)), "
                           "s1=log((1+e)/2); d=s/2; d1>c clipped; K=d0+c; CE=log 2; "
                           "S=(s0+1)/2; g0=-lam/2+(1-lam)/2*(s0+1-S); g1=lam/2-(1-lam)/2*S")


def case_temperature_v3():
    # D = [2, 0, 0], T = [0, 0, 0], tau = 2, lambda = 0, c = inf.
    # q = (e, 1, 1)/(e+2), p = (1/3, 1/3, 1/3).
    tau = 2.0
    Z = E + 2
    q = [E / Z, 1 / Z, 1 / Z]
    s = [math.log(3 * E / Z), math.log(3 / Z), math.log(3 / Z)]
    rkl = math.log(3) + E / Z - math.log(Z)
    # with lambda = 0 and no clipping: S = 1 + RKL and g_u = (1/tau) q_u (s_u - RKL)
    g = [q[u] * (s[u] - rkl) / tau for u in range(3)]
    ce = math.log(Z) - 1.0                 # y = argmax T = 0 (all tied -> lowest id)
    return dict(name="temperature_v3", D=[2.0, 0.0, 0.0], T=[0.0, 0.0, 0.0], tau=tau, lam=0.0,
                clip_c="inf", loss=rkl, rkl=rkl, kc=rkl, ce=ce, grad=g,
                derivation="q=(e,1,1)/(e+2), p=1/3; RKL=log3+e/(e+2)-log(e+2); "
                           "g_u=q_u(s_u-RKL)/tau; CE=-log q0=log(e+2)-1")


def case_equal_rows():
    # D = T = [1, -1, 0.5, 0.5]: q = p, so every d_v = 0, K_c = 0 for any c >= 0, and with
    # lambda = 0 the gradient vanishes.
    return dict(name="equal_rows", D=[1.0, -1.0, 0.5, 0.5], T=[1.0, -1.0, 0.5, 0.5], tau=1.0,
                lam=0.0, clip_c=0.01, loss=0.0, rkl=0.0, kc=0.0,
                ce=math.log(E + math.exp(-1) + 2 * math.exp(0.5)) - 1.0, grad=[0.0] * 4,
                derivation="q=p => s=0, d=0, K=0, S=1, g=q(s+1-S)=0; CE=lse-1")


def main():
    cases = [case_clip_v2(), case_temperature_v3(), case_equal_rows()]
    out = dict(source="hand-derived closed forms (the pages print no worked example)",
               cases=cases)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
