"""Hymba hybrid-head mixer on B200 (sm_100a): C-ABI library ``libhymba.so`` plus a thin
ctypes binding.  Importing the package loads nothing; the binding loads the library on
first use and raises if it is missing."""
