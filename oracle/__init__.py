"""CPU oracle for HGA routed attention.

Test infrastructure only: imported by tests/, the smoke check and the
benchmark's CPU-baseline leg, never by the product package.
"""
