// Status bits shared by host and device code (values from the public header).
#pragma once
#include "../../include/mla.h"
