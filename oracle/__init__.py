"""Plain CPU oracle for the D-Quant hot path (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline/reference
legs may import this package. The product package never imports it.
"""
