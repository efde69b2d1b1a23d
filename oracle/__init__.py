"""CPU oracle for the BATQuant W4A4 MXFP4 path -- test infrastructure only.

Imported by the tests, the smoke check and the benchmark's CPU-baseline arm;
never by the product library.
"""
